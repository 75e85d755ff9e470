"""Attention over other KV cache layouts against the float64 oracle on the same bytes:
mixed-precision rows (csa_sparse_mqa_mixed_kv, hca_dense_mqa_mixed_kv) and paged caches
(csa_sparse_mqa_paged, hca_dense_mqa_paged); and the indexer over paged keys
(csa_index_topk_paged: FP8, bf16 and MXFP4 keys), which must give exactly the scores and
selection of the contiguous keys.

For mixed rows the workloads' bf16 caches are re-encoded by the input encoder (the first
c - r values as e4m3 with a row scale, the RoPE values as bf16); the oracle decodes those
bytes exactly, and the kernel widens code * scale to bf16 before its tensor-core products.
For paged caches the rows are scattered into a pool of pages through a shuffled page
table, and the oracle reads the contiguous cache. The outputs must meet the bf16 output
tolerance.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_08_b200 as csa
from long_context_sparse_08_b200 import runner as R
from long_context_sparse_08_b200 import workloads as W
from oracle import pipeline as P
import tests.parity_util as U

pytestmark = [
    pytest.mark.gpu,
]


def _mixed(name):
    s, inp = U.inputs(name)
    kv = W.bf16_bits_to_f32(inp["kv_cache"])
    codes, scale, rope = W.quant_mixed_kv(kv, s.rope_dims)
    rows = np.concatenate([codes, rope.view(np.uint8)], axis=-1)  # c + r bytes per row
    inp2 = {k: v for k, v in inp.items() if k != "kv_cache"}
    inp2.update(kv_codes=codes, kv_scale=scale, kv_rope=rope)
    return s, inp, inp2, torch.from_numpy(np.ascontiguousarray(rows)).cuda(), \
        torch.from_numpy(scale).cuda()


@pytest.mark.parametrize("name", ["mid_decode_fp8", "mid_decode_mxfp4", "edge_decode_bf16"])
def test_sparse_mqa_over_mixed_rows(name):
    s, inp, inp2, rows, scale = _mixed(name)
    res = P.run(s, inp2, want_scores=False)
    dev = R.upload(inp, s)
    idx = np.full((s.B, s.T, s.topk), -1, np.int32)
    for (b, ti), sel in res["idx"].items():
        idx[b, ti] = sel
    p = R.params_for(s)
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_SPARSE_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    csa.csa_sparse_mqa_mixed_kv(p, s.B, s.T, dev["q"], dev["q_pos"], rows, scale, s.n_cap,
                                torch.from_numpy(idx).cuda(), dev["win_kv"],
                                dev["win_kv"].shape[1], dev["win_pos0"], dev["sink"], None, out,
                                ws, ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = out.float().cpu().numpy()
    for (b, ti), ref in res["out"].items():
        U.check_out(got[b, ti], ref, "bf16", f"{name} mixed KV b={b} t={ti}")


@pytest.mark.parametrize("name", ["mid_hca_decode", "edge_hca_decode", "long_hca_decode"])
def test_dense_mqa_over_mixed_rows(name):
    s, inp, inp2, rows, scale = _mixed(name)
    res = P.run(s, inp2)
    dev = R.upload(inp, s)
    p = R.params_for(s)
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    csa.hca_dense_mqa_mixed_kv(p, s.B, s.T, dev["q"], dev["q_pos"], rows, scale, s.n_cap,
                               dev["win_kv"], dev["win_kv"].shape[1], dev["win_pos0"],
                               dev["sink"], None, out, ws, ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = out.float().cpu().numpy()
    for (b, ti), ref in res["out"].items():
        U.check_out(got[b, ti], ref, "bf16", f"{name} mixed KV b={b}")


def _paged(cache, page_rows, seed, extra_pages=5):
    """Scatter a contiguous cache [B, n_cap, ...] into a page pool through a shuffled page
    table; returns (pool, table [B, max_pages] int32)."""
    B, n_cap = cache.shape[:2]
    assert n_cap % page_rows == 0
    max_pages = n_cap // page_rows
    n_pages = B * max_pages + extra_pages
    perm = np.random.default_rng(seed).permutation(n_pages).astype(np.int32)
    table = perm[:B * max_pages].reshape(B, max_pages)
    pool = np.zeros((n_pages, page_rows) + cache.shape[2:], cache.dtype)
    for b in range(B):
        for lp in range(max_pages):
            pool[table[b, lp]] = cache[b, lp * page_rows:(lp + 1) * page_rows]
    return pool, np.ascontiguousarray(table)


def _dev(a):
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()


@pytest.mark.parametrize("name,mixed,page_rows", [("mid_decode_fp8", False, 32),
                                                  ("mid_decode_mxfp4", True, 32),
                                                  ("edge_decode_bf16", False, 32)])
def test_sparse_mqa_over_paged_cache(name, mixed, page_rows):
    s, inp = U.inputs(name)
    if mixed:
        s, inp, inp2, _, _ = _mixed(name)
        codes, rope = inp2["kv_codes"], inp2["kv_rope"]
        rows = np.concatenate([codes, rope.view(np.uint8)], axis=-1)
        pool, table = _paged(rows, page_rows, 3)
        spool, _ = _paged(inp2["kv_scale"][..., None], page_rows, 3)
        scales = _dev(spool[..., 0])
    else:
        inp2 = inp
        pool, table = _paged(inp["kv_cache"], page_rows, 3)
        scales = None
    res = P.run(s, inp2, want_scores=False)
    dev = R.upload(inp, s)
    idx = np.full((s.B, s.T, s.topk), -1, np.int32)
    for (b, ti), sel in res["idx"].items():
        idx[b, ti] = sel
    p = R.params_for(s)
    fmt = csa.CSA_MIXED_FP8_BF16 if mixed else csa.CSA_BF16
    pool_d, table_d = _dev(pool), _dev(table)
    kv = csa.paged_kv(fmt, pool_d, scales, table_d, pool.shape[0], page_rows, table.shape[1])
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_SPARSE_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    csa.csa_sparse_mqa_paged(p, s.B, s.T, dev["q"], dev["q_pos"], kv,
                             torch.from_numpy(idx).cuda(), dev["win_kv"], dev["win_kv"].shape[1],
                             dev["win_pos0"], dev["sink"], None, out, ws, ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = out.float().cpu().numpy()
    for (b, ti), ref in res["out"].items():
        U.check_out(got[b, ti], ref, "bf16", f"{name} paged b={b} t={ti}")


@pytest.mark.parametrize("name,page_rows", [("mid_hca_decode", 1), ("mid_hca_decode", 8),
                                            ("long_hca_decode", 8)])
def test_dense_mqa_over_paged_cache(name, page_rows):
    s, inp = U.inputs(name)
    res = P.run(s, inp)
    dev = R.upload(inp, s)
    pool, table = _paged(inp["kv_cache"], page_rows, 4)
    p = R.params_for(s)
    kv = csa.paged_kv(csa.CSA_BF16, _dev(pool), None, _dev(table), pool.shape[0], page_rows,
                      table.shape[1])
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    csa.hca_dense_mqa_paged(p, s.B, s.T, dev["q"], dev["q_pos"], kv, dev["win_kv"],
                            dev["win_kv"].shape[1], dev["win_pos0"], dev["sink"], None, out, ws,
                            ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = out.float().cpu().numpy()
    for (b, ti), ref in res["out"].items():
        U.check_out(got[b, ti], ref, "bf16", f"{name} paged({page_rows}) b={b}")


def test_paged_cache_with_a_bad_page_id_reports_it():
    s, inp = U.inputs("mid_hca_decode")
    dev = R.upload(inp, s)
    pool, table = _paged(inp["kv_cache"], 8, 5)
    table[0, 0] = pool.shape[0]  # outside the pool
    p = R.params_for(s)
    kv = csa.paged_kv(csa.CSA_BF16, _dev(pool), None, _dev(table), pool.shape[0], 8,
                      table.shape[1])
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    csa.device_error()
    csa.hca_dense_mqa_paged(p, s.B, s.T, dev["q"], dev["q_pos"], kv, dev["win_kv"],
                            dev["win_kv"].shape[1], dev["win_pos0"], dev["sink"], None, out, ws,
                            ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 205


@pytest.mark.parametrize("name", ["edge_decode_fp8_tc", "edge_decode_bf16_tc",
                                  "mid_prefill_bf16_tc", "edge_decode_mxfp4",
                                  "edge_decode_mxfp4_long", "mid_decode_mxfp4_sel"])
@pytest.mark.parametrize("bf16_scores", [0, 1])
@pytest.mark.parametrize("holes", [False, True], ids=["all_pages", "unallocated_tail"])
def test_index_topk_over_paged_keys_equals_contiguous(name, bf16_scores, holes):
    """With `holes`, the table entries of pages past a request's visible keys are -1 (pages
    not yet allocated): the indexer must not read them, nor report a bad page id."""
    s, inp = U.inputs(name)
    dev = R.upload(inp, s)
    p = R.params_for(s)
    kdt = csa.DTYPES[s.idx]
    B, T, N = s.B, s.T, s.n_cap
    entry = csa.CSA_WS_INDEX_TOPK_BF16 if bf16_scores else csa.CSA_WS_INDEX_TOPK
    need = csa.workspace_size(p, entry, kdt, B, T, N)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    sdt = torch.int16 if bf16_scores else torch.float32
    idx_c = torch.empty((B, T, s.topk), dtype=torch.int32, device="cuda")
    sc_c = torch.zeros((B, T, N), dtype=sdt, device="cuda")
    if bf16_scores:
        csa.csa_index_topk_bf16(p, kdt, B, T, N, dev["qI"], dev.get("qI_scale"), dev["w"],
                                dev["KI"], dev.get("KI_scale"), dev["q_pos"], idx_c, sc_c, ws,
                                need)
    else:
        csa.csa_index_topk(p, kdt, B, T, N, dev["qI"], dev.get("qI_scale"), dev["w"], dev["KI"],
                           dev.get("KI_scale"), dev["q_pos"], idx_c, sc_c, ws, need)
    pool, table = _paged(inp["KI"], 128, 6)
    if holes:
        for b in range(B):
            nv = int(max(0, min(int(inp["q_pos"][b].max()) // s.m, N)))
            table[b, -(-nv // 128):] = -1
    scales = None
    if "KI_scale" in inp:
        spool, _ = _paged(inp["KI_scale"][..., None], 128, 6)
        scales = _dev(np.ascontiguousarray(spool[..., 0]))
    keys = csa.paged_kv(kdt, _dev(pool), scales, _dev(table), pool.shape[0], 128, table.shape[1])
    idx_p = torch.empty_like(idx_c)
    sc_p = torch.zeros_like(sc_c)
    torch.cuda.synchronize()
    csa.device_error()
    csa.csa_index_topk_paged(p, B, T, keys, dev["qI"], dev.get("qI_scale"), dev["w"],
                             dev["q_pos"], bf16_scores, idx_p, sc_p, ws, need)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    assert torch.equal(idx_p, idx_c)
    pos = inp["q_pos"]
    for b in range(B):
        for t in range(T):
            n = int(max(0, min(pos[b, t] // s.m, N)))
            assert torch.equal(sc_p[b, t, :n], sc_c[b, t, :n]), f"{name} b={b} t={t}"


def _paged_forward(s, inp, dev, kv_fmt, kv_rows, kv_scale, bf16_scores, ring=None):
    """csa_forward_paged over KV pages of 32 rows and key pages of 128 rows (shuffled); with
    `ring` ([B, n_win, c] device rows) the window is read as the state cache's ring."""
    p = R.params_for(s)
    B, T, N = s.B, s.T, s.n_cap
    kv_pool, kv_table = _paged(kv_rows, 32, 7)
    kvs = None
    if kv_scale is not None:
        sp, _ = _paged(kv_scale[..., None], 32, 7)
        kvs = _dev(np.ascontiguousarray(sp[..., 0]))
    k_pool, k_table = _paged(inp["KI"], 128, 8)
    ks = None
    if "KI_scale" in inp:
        sp, _ = _paged(inp["KI_scale"][..., None], 128, 8)
        ks = _dev(np.ascontiguousarray(sp[..., 0]))
    kv = csa.paged_kv(kv_fmt, _dev(kv_pool), kvs, _dev(kv_table), kv_pool.shape[0], 32,
                      kv_table.shape[1])
    keys = csa.paged_kv(csa.DTYPES[s.idx], _dev(k_pool), ks, _dev(k_table), k_pool.shape[0], 128,
                        k_table.shape[1])
    need = csa.workspace_size(p, csa.CSA_WS_FORWARD, csa.DTYPES[s.idx], B, T, N)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    idx = torch.empty((B, T, s.topk), dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, T, N), dtype=torch.int16 if bf16_scores else torch.float32,
                     device="cuda")
    torch.cuda.synchronize()
    csa.device_error()
    win, L, pos0 = (dev["win_kv"], dev["win_kv"].shape[1], dev["win_pos0"]) if ring is None \
        else (ring, ring.shape[1], None)
    csa.csa_forward_paged(p, B, T, kv, keys, bf16_scores, dev["qI"], dev.get("qI_scale"),
                          dev["w"], dev["q"], None, dev["q_pos"], win, L, pos0, dev["sink"], idx,
                          sc, out, ws, need)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    return out, idx, sc


@pytest.mark.parametrize("name", ["edge_decode_fp8_tc", "edge_decode_bf16_tc",
                                  "edge_decode_mxfp4", "mid_decode_mxfp4_sel"])
def test_forward_paged_equals_contiguous(name):
    s, inp = U.inputs(name)
    dev = R.upload(inp, s)
    st = R.Step(s, dev, want_scores=True)
    st()
    torch.cuda.synchronize()
    out, idx, sc = _paged_forward(s, inp, dev, csa.CSA_BF16, inp["kv_cache"], None, 0)
    assert torch.equal(idx, st.out_idx)
    assert torch.equal(out, st.out)


@pytest.mark.parametrize("name", ["edge_decode_fp8_tc", "edge_decode_bf16_tc"])
def test_forward_paged_bf16_scores_over_mixed_kv(name):
    s, inp, inp2, _, _ = _mixed(name)
    dev = R.upload(inp, s)
    codes, rope = inp2["kv_codes"], inp2["kv_rope"]
    rows = np.concatenate([codes, rope.view(np.uint8)], axis=-1)
    out, idx, sc = _paged_forward(s, inp, dev, csa.CSA_MIXED_FP8_BF16, rows, inp2["kv_scale"], 1)
    idx = idx.cpu().numpy()
    got16 = sc.cpu().numpy().view(np.uint16)
    res = P.run(s, inp2, want_scores=True)
    from oracle import csa_oracle as O
    import tests.test_bf16_scores as BS

    for (b, ti), ref in res["scores"].items():
        g = O.dec_bf16(got16[b, ti, :ref.size])
        BS._valid_selection(idx[b, ti], g, s.topk)
    sel = {(b, ti): idx[b, ti] for (b, ti) in res["out"]}
    ref_out = P.run(s, inp2, list(sel), idx_override=sel, want_scores=False)["out"]
    got = out.float().cpu().numpy()
    for (b, ti), r in ref_out.items():
        U.check_out(got[b, ti], r, "bf16", f"{name} paged mixed b={b} t={ti}")


@pytest.mark.parametrize("name", ["edge_decode_fp8_tc", "edge_decode_bf16_tc"])
def test_forward_paged_reads_the_window_ring(name):
    """The state cache's window ring (position p in row p mod n_win) gives the same output as
    the linear window buffer."""
    s, inp = U.inputs(name)
    dev = R.upload(inp, s)
    win = inp["win_kv"]
    ring = np.zeros((s.B, s.n_win, s.c), win.dtype)
    for b in range(s.B):
        t, p0 = int(inp["q_pos"][b, 0]), int(inp["win_pos0"][b])
        for pos in range(max(t - s.n_win + 1, 0), t + 1):
            ring[b, pos % s.n_win] = win[b, pos - p0]
    out_l, idx_l, _ = _paged_forward(s, inp, dev, csa.CSA_BF16, inp["kv_cache"], None, 0)
    out_r, idx_r, _ = _paged_forward(s, inp, dev, csa.CSA_BF16, inp["kv_cache"], None, 0,
                                     ring=_dev(ring))
    assert torch.equal(idx_r, idx_l)
    assert torch.equal(out_r, out_l)

