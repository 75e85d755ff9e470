"""A decode step over the state cache, end to end, against the float64 oracle.

Three requests feed their tokens one at a time to csa_state_append: the KV entries go into
pages of 32 entries (bf16), the compressed indexer keys into pages of 128 keys (MXFP4, the
FP4 indexer cache of 【论文解读】DeepSeek-V4 二(四) and 二(六)) and the window rows into the
ring. One csa_forward_paged call at every request's last position then runs index -> top-k
-> sparse MQA over the pools. Page tables are shuffled, and the entries of pages nothing has
been written to yet are -1.

The oracle feeds the same raw rows through its own state cache (oracle/state_cache.py),
stores the finished entries with the input encoders (bf16; MXFP4), and runs its indexer and
attention on those. Checks:
  - KV pages: every entry within one bf16 rounding of the oracle's;
  - key pages: the MXFP4 bytes equal the encoder's bytes of the oracle's keys, except where
    the fp32 key lies within fp32 error of an e2m1 / exponent rounding boundary (at most 1%
    of the keys; such keys are left out of the score checks);
  - index scores within 1e-4 relative (floored at 1e-3 of the row's largest score), or, for
    a score that signed head weights cancel, within 1e-4 of the sum of the magnitudes of its
    terms (parity_util.score_limit; BF16 scores: plus one bf16 rounding);
  - the selection: valid for the scores the GPU stored, and equal to the oracle's except at
    near-ties of the k-th score;
  - the output: the oracle's attention over the GPU's selection, within the bf16 output
    tolerance.
The N_cap = 8192 case takes the decode top-k (histogram filled by the indexer), 1024 the
row top-k. In the prefill cases request 1 starts from a prefill chunk of 302 tokens handed
over with csa_compress_paged / csa_compress + csa_encode_paged and csa_state_resume, and then
decodes; the oracle takes every token one at a time. One case stores the KV entries as mixed-precision rows (e4m3 with a row scale,
bf16 RoPE dims; 一(三)4): they must decode to within one step of each format of the
oracle's entries, and the oracle attends its own mixed rows. The HCA case (m' = 128, pages
of one entry, hca_dense_mqa_paged over the ring) attends every visible entry.
"""
import math

import numpy as np
import pytest

from oracle import csa_oracle as O
from oracle import state_cache as SC
from long_context_sparse_08_b200 import workloads as W
import tests.parity_util as U

pytestmark = [
    pytest.mark.gpu,
]

M, C, R, D_I, H, H_I, K, N_WIN = 4, 512, 64, 128, 64, 64, 64, 128
BASE, EPS = 10000.0, 1e-6
KV_ROWS, KEY_ROWS = 32, 128  # entries per page
N_TOK = (1100, 517, 2051)    # tokens each request appends (129 visible keys: a page and one)
PREFILL = 302                # with a prefill, request 1's first tokens come as one chunk


class Stream:
    """Seeded raw rows, queries and page tables of the three requests (host arrays)."""

    def __init__(self, n_cap, seed=2026):
        self.B, self.n_cap = len(N_TOK), n_cap
        n = max(N_TOK)
        self.kv = W.make_state_stream(B=self.B, n_tok=n, m=M, c=C, overlap=1, io="bf16",
                                      seed=seed)
        self.key = W.make_state_stream(B=self.B, n_tok=n, m=M, c=D_I, overlap=1, io="bf16",
                                       seed=seed + 1)
        g = np.random.default_rng(seed + 2)
        self.q = W.f32_to_bf16_bits(g.standard_normal((self.B, 1, H, C), np.float32))
        qI = g.standard_normal((self.B, 1, H_I, D_I), np.float32)
        self.qI, self.qI_scale = W.quant_mxfp4(qI)
        self.w = g.standard_normal((self.B, 1, H_I), np.float32)
        self.sink = g.standard_normal((H,), np.float32)
        self.pos = np.array([[t - 1] for t in N_TOK], np.int64)
        self.kv_table, self.n_kv_pages = self._table(KV_ROWS, g)
        self.key_table, self.n_key_pages = self._table(KEY_ROWS, g)

    def _table(self, rows, g):
        """Shuffled page table [B, n_cap / rows]: the pages a request's entries fill, in a
        pool with 3 spare pages; -1 past them."""
        max_pages = self.n_cap // rows
        used = [-(-(t // M) // rows) for t in N_TOK]
        n_pages = sum(used) + 3
        perm = g.permutation(n_pages).astype(np.int32)
        table = np.full((self.B, max_pages), -1, np.int32)
        k = 0
        for b, u in enumerate(used):
            table[b, :u] = perm[k:k + u]
            k += u
        return table, n_pages

    def n_vis(self, b):
        return O.visible_entries(int(self.pos[b, 0]), M, self.n_cap)


def stored_kv(kv_f64, kv_fmt):
    """The oracle's entries as the cache stores them (input encoders), decoded."""
    x = kv_f64.astype(np.float32)
    if kv_fmt == "mixed":
        return O.dec_mixed_kv(*W.quant_mixed_kv(x, R))
    return O.dec_bf16(W.f32_to_bf16_bits(x))


def oracle_caches(st: Stream, kv_fmt="bf16"):
    """Per request: the oracle's KV entries (as stored, decoded), its fp32-cast keys, the
    MXFP4 bytes the encoder makes of them, and those keys decoded."""
    out = []
    for b, n in enumerate(N_TOK):
        caches = []
        for src, c, fin, rows in ((st.kv, C, True, KV_ROWS), (st.key, D_I, False, KEY_ROWS)):
            pool = SC.PagePool(-(-(n // M) // rows) + 1, rows, c)
            cs = SC.CsaState(pool, m=M, c=c, bias=O.dec_bf16(src["bias"]), n_win=N_WIN, r=R,
                             base=BASE, eps=EPS, block_tokens=M * rows, finalize=fin)
            r = {k: O.dec_bf16(src[k][b, :n]) for k in ("Ca", "Cb", "Za", "Zb", "win")}
            for t in range(n):
                cs.append(r["Ca"][t], r["Cb"][t], r["Za"][t], r["Zb"][t], r["win"][t])
            caches.append(cs.entries())
        kv, keys = caches
        packed, ex = W.quant_mxfp4(keys.astype(np.float32))
        out.append(dict(kv_f64=kv, kv=stored_kv(kv, kv_fmt), keys_packed=packed, keys_ex=ex,
                        keys=O.dec_mxfp4(packed, ex), win=O.dec_bf16(st.kv["win"][b, :n])))
    return out


def _up(x):
    import torch

    a = np.ascontiguousarray(x)
    return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()


def prefill_request(csa, torch, b, p_kv, p_key, kv_src, key_src, kv_desc, key_desc, kv_state,
                    key_state, ring, mixed):
    """Request b's first PREFILL tokens as a prefill chunk: the entries of its complete blocks
    into the pages (bf16 KV: csa_compress_paged; mixed KV and MXFP4 keys: csa_compress in
    fp32, then csa_encode_paged), then its raw tail and window into the state cache
    (csa_state_resume)."""
    n_full = PREFILL - PREFILL % M
    f32 = lambda t: t.view(torch.bfloat16).float().contiguous()  # noqa: E731  (exact)
    chunk = lambda src, k: src[k][b:b + 1, :n_full]  # noqa: E731
    if not mixed:
        csa.csa_compress_paged(p_kv, csa.CSA_BF16, 1, n_full, 0, chunk(kv_src, "Ca"),
                               chunk(kv_src, "Cb"), chunk(kv_src, "Za"), chunk(kv_src, "Zb"),
                               kv_src["bias"], None, None, None, 1, kv_desc)
    for p, src, fin, desc, c, use in ((p_kv, kv_src, 1, kv_desc, C, mixed),
                                      (p_key, key_src, 0, key_desc, D_I, True)):
        if not use:
            continue
        tmp = torch.zeros((1, n_full // M, c), dtype=torch.float32, device="cuda")
        csa.csa_compress(p, csa.CSA_F32, 1, n_full, 0, n_full // M, f32(chunk(src, "Ca")),
                         f32(chunk(src, "Cb")), f32(chunk(src, "Za")), f32(chunk(src, "Zb")),
                         f32(src["bias"]), None, None, None, fin, tmp)
        csa.csa_encode_paged(p, csa.CSA_F32, 1, n_full // M, 0, tmp, desc)
    tail = lambda src, k: src[k][b:b + 1, :PREFILL]  # noqa: E731
    csa.csa_state_resume(p_kv, csa.CSA_BF16, 1, 0, PREFILL, tail(kv_src, "Ca"),
                         tail(kv_src, "Cb"), tail(kv_src, "Za"), tail(kv_src, "Zb"),
                         tail(kv_src, "win"), kv_state[b:b + 1], ring[b:b + 1])
    csa.csa_state_resume(p_key, csa.CSA_BF16, 1, 0, PREFILL, tail(key_src, "Ca"),
                         tail(key_src, "Cb"), tail(key_src, "Za"), tail(key_src, "Zb"), None,
                         key_state[b:b + 1], None)


def run_gpu(st: Stream, bf16_scores: int, kv_fmt="bf16", prefill=False):
    """The appends (after a prefill chunk for request 1 when `prefill`) and the forward call;
    returns host copies of the pools and the results."""
    import torch
    import long_context_sparse_08_b200 as csa

    up = _up
    torch.cuda.synchronize()
    csa.device_error()
    B = st.B
    mixed = kv_fmt == "mixed"
    p_kv = csa.make_params(m=M, overlap=1, c=C, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                           n_heads=H, n_idx_heads=H_I, d_idx=D_I, topk=K, n_win=N_WIN)
    p_key = csa.make_params(m=M, overlap=1, c=D_I, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                            n_win=N_WIN)
    kv_pages = torch.zeros((st.n_kv_pages, KV_ROWS, C + R), dtype=torch.uint8, device="cuda") \
        if mixed else torch.zeros((st.n_kv_pages, KV_ROWS, C), dtype=torch.int16, device="cuda")
    kv_scales = torch.zeros((st.n_kv_pages, KV_ROWS), dtype=torch.float32, device="cuda") \
        if mixed else None
    kv_out = csa.CSA_MIXED_FP8_BF16 if mixed else csa.CSA_BF16
    key_pages = torch.zeros((st.n_key_pages, KEY_ROWS, D_I // 2), dtype=torch.uint8,
                            device="cuda")
    key_ex = torch.zeros((st.n_key_pages, KEY_ROWS, 4), dtype=torch.uint8, device="cuda")
    kv_state = torch.zeros((B, 2 * M, 4, C), dtype=torch.int16, device="cuda")
    key_state = torch.zeros((B, 2 * M, 4, D_I), dtype=torch.int16, device="cuda")
    ring = torch.zeros((B, N_WIN, C), dtype=torch.int16, device="cuda")
    kv_table, key_table = up(st.kv_table), up(st.key_table)
    kv_src = {k: up(st.kv[k]) for k in st.kv}
    key_src = {k: up(st.key[k]) for k in st.key}
    for b, n in enumerate(N_TOK):  # one request per call, its own state / ring / table rows
        # every pointer 16-byte aligned: the position in a 16-byte row, the table row a copy
        pos_all = torch.zeros((n, 2), dtype=torch.int64, device="cuda")
        pos_all[:, 0] = torch.arange(n, device="cuda")
        kv_tb, key_tb = up(st.kv_table[b:b + 1]), up(st.key_table[b:b + 1])
        t0 = 0
        if prefill and b == 1:
            kv_desc = csa.paged_kv(kv_out, kv_pages, kv_scales, kv_tb, st.n_kv_pages, KV_ROWS,
                                   kv_table.shape[1])
            key_desc = csa.paged_kv(csa.CSA_MXFP4, key_pages, key_ex, key_tb, st.n_key_pages,
                                    KEY_ROWS, key_table.shape[1])
            prefill_request(csa, torch, b, p_kv, p_key, kv_src, key_src, kv_desc, key_desc,
                            kv_state, key_state, ring, mixed)
            t0 = PREFILL
        for t in range(t0, n):
            pos = pos_all[t, :1]
            r = {k: v[b, t:t + 1] for k, v in kv_src.items() if k != "bias"}
            csa.csa_state_append(p_kv, csa.CSA_BF16, 1, pos, r["Ca"], r["Cb"], r["Za"], r["Zb"],
                                 r["win"], kv_src["bias"], None, 1, kv_state[b:b + 1],
                                 ring[b:b + 1], kv_out, kv_pages, kv_scales, st.n_kv_pages,
                                 KV_ROWS, kv_tb, kv_table.shape[1])
            r = {k: v[b, t:t + 1] for k, v in key_src.items() if k != "bias"}
            csa.csa_state_append(p_key, csa.CSA_BF16, 1, pos, r["Ca"], r["Cb"], r["Za"],
                                 r["Zb"], None, key_src["bias"], None, 0, key_state[b:b + 1],
                                 None, csa.CSA_MXFP4, key_pages, key_ex, st.n_key_pages,
                                 KEY_ROWS, key_tb, key_table.shape[1])
    torch.cuda.synchronize()
    assert csa.device_error() == 0, "appends"
    kv = csa.paged_kv(kv_out, kv_pages, kv_scales, kv_table, st.n_kv_pages, KV_ROWS,
                      kv_table.shape[1])
    keys = csa.paged_kv(csa.CSA_MXFP4, key_pages, key_ex, key_table, st.n_key_pages, KEY_ROWS,
                        key_table.shape[1])
    need = csa.workspace_size(p_kv, csa.CSA_WS_FORWARD, csa.CSA_MXFP4, B, 1, st.n_cap)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, 1, H, C), dtype=torch.int16, device="cuda")
    idx = torch.empty((B, 1, K), dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, 1, st.n_cap), dtype=torch.int16 if bf16_scores else torch.float32,
                     device="cuda")
    args = (up(st.qI), up(st.qI_scale), up(st.w), up(st.q), None, up(st.pos), ring, N_WIN, None,
            up(st.sink))
    csa.csa_forward_paged(p_kv, B, 1, kv, keys, bf16_scores, *args, idx, sc, out, ws, need)
    # a second run into fresh buffers must agree bit for bit (fixed-order combine, index
    # tie-break: a race would show as a difference)
    idx2, sc2, out2 = torch.empty_like(idx), torch.zeros_like(sc), torch.empty_like(out)
    csa.csa_forward_paged(p_kv, B, 1, kv, keys, bf16_scores, *args, idx2, sc2, out2, ws, need)
    torch.cuda.synchronize()
    assert csa.device_error() == 0, "forward"
    assert torch.equal(idx, idx2) and torch.equal(sc, sc2) and torch.equal(out, out2)
    scores = sc.cpu().numpy()
    scores = O.dec_bf16(scores.view(np.uint16)) if bf16_scores else scores.astype(np.float64)
    kvp = kv_pages.cpu().numpy()
    return dict(kv_pages=kvp if mixed else kvp.view(np.uint16),
                kv_scales=None if kv_scales is None else kv_scales.cpu().numpy(),
                key_pages=key_pages.cpu().numpy(), key_ex=key_ex.cpu().numpy(),
                idx=idx.cpu().numpy(), scores=scores,
                out=O.dec_bf16(out.cpu().numpy().view(np.uint16)))


def page_rows_of(table, rows, b, n):
    """(page, slot) of entries 0 .. n-1 of request b."""
    i = np.arange(n)
    return table[b, i // rows], i % rows


def check_kv_rows(got_rows, got_scales, ref, kv_fmt, what):
    """Stored KV entries against the oracle's fp64 entries: within the fp32 error and one
    rounding of the storage format."""
    if kv_fmt != "mixed":
        U.check_rows(O.dec_bf16(got_rows), ref, "bf16", what)
        return
    r0 = C - R
    dq = O.dec_mixed_kv(got_rows[:, :r0], got_scales,
                        np.ascontiguousarray(got_rows[:, r0:]).view(np.uint16))
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    # half an e4m3 step (2^-4 of |x|, 2^-10 x scale below the normal range); half a bf16 ulp
    bound = np.concatenate([
        np.maximum(np.abs(ref[:, :r0]) * 2.0 ** -4, got_scales[:, None] * 2.0 ** -10) * 1.01,
        np.abs(ref[:, r0:]) * 2.0 ** -8 * 1.01], axis=1) + 2e-4 * rms
    assert np.all(np.abs(dq - ref) <= bound), f"{what}: mixed rows"


def check_pages(st, ora, got, kv_fmt="bf16"):
    """KV entries within one rounding of their format; key bytes equal except near rounding
    boundaries. Returns, per request, the keys whose stored bytes differ from the oracle's."""
    off = []
    for b, n in enumerate(N_TOK):
        o = ora[b]
        ne = n // M
        pg, sl = page_rows_of(st.kv_table, KV_ROWS, b, ne)
        check_kv_rows(got["kv_pages"][pg, sl],
                      None if got["kv_scales"] is None else got["kv_scales"][pg, sl],
                      o["kv_f64"], kv_fmt, f"request {b}: KV entries")
        pg, sl = page_rows_of(st.key_table, KEY_ROWS, b, ne)
        packed = got["key_pages"][pg, sl]
        ex = np.stack([O.unblock_key_scales(got["key_ex"][p])[s] for p, s in zip(pg, sl)])
        bad = np.flatnonzero(np.any(packed != o["keys_packed"], axis=1) |
                             np.any(ex != o["keys_ex"], axis=1))
        assert bad.size <= max(1, ne // 100), f"request {b}: {bad.size} keys stored differently"
        # a differing key is still the same key to within one e2m1 step of its block
        if bad.size:
            dq = O.dec_mxfp4(packed[bad], ex[bad])
            step = np.repeat(np.exp2(o["keys_ex"][bad].astype(np.float64) - 126.0), 32, axis=1)
            assert np.all(np.abs(dq - o["keys"][bad]) <= 2 * step), f"request {b}: key codes"
        off.append(set(bad.tolist()))
    return off


def check_selection_and_output(st, ora, got, off, bf16_scores):
    qI = O.dec_mxfp4(st.qI, st.qI_scale)
    for b in range(st.B):
        o, t, nv = ora[b], int(st.pos[b, 0]), st.n_vis(b)
        ref = O.index_scores(qI[b, 0], st.w[b, 0], o["keys"], nv)
        scale = O.index_score_scale(qI[b, 0], st.w[b, 0], o["keys"], nv)
        g = got["scores"][b, 0, :nv]
        ok = np.array([s not in off[b] for s in range(nv)], bool)
        lim = U.score_limit(ref, scale)[0] + (U.bf16_ulp(ref) if bf16_scores else 0.0)
        assert np.all(np.abs(g - ref)[ok] <= lim[ok]), f"request {b}: index scores"
        sel = got["idx"][b, 0]
        kk = min(K, nv)
        assert np.all(sel[kk:] == -1) and len(set(sel[:kk].tolist())) == kk
        # valid for the GPU's own scores: larger first, ties by index, nothing larger left out
        gs = g.astype(np.float64)
        for j in range(kk - 1):
            a, c = gs[sel[j]], gs[sel[j + 1]]
            assert a > c or (a == c and sel[j] < sel[j + 1]), f"request {b}: order at {j}"
        if kk < nv:
            last = gs[sel[kk - 1]]
            assert last >= np.delete(gs, sel[:kk]).max(), f"request {b}: k-th"
            tied = np.flatnonzero(gs == last)  # among equal values the smaller indices win
            n_tied = int(np.sum(gs[sel[:kk]] == last))
            assert sorted(sel[:kk][gs[sel[:kk]] == last].tolist()) == tied[:n_tied].tolist()
        # against the oracle: different only at near-ties of the k-th score (or at a key
        # stored differently)
        theirs = (O.topk_select_bf16 if bf16_scores else O.topk_select)(ref, K)[:kk]
        tau = (O.round_to_bf16(ref) if bf16_scores else ref)[theirs[-1]]
        tol = 1e-4 * max(abs(tau), 1e-3 * np.abs(ref).max()) + \
            (U.bf16_ulp(np.array([tau]))[0] if bf16_scores else 0.0)
        for i in set(sel[:kk].tolist()).symmetric_difference(theirs.tolist()):
            assert i in off[b] or abs(ref[i] - tau) <= tol, f"request {b}: {i} not a near-tie"
        # the oracle's attention over the GPU's selection
        want = O.csa_query(O.dec_bf16(st.q[b, 0]), t, o["kv"], sel, o["win"], 0, st.sink, r=R,
                           base=BASE, eps=EPS, scale=1.0 / math.sqrt(C), n_win=N_WIN)
        U.check_out(got["out"][b, 0], want, "bf16", f"request {b}: output")


CASES = [(1024, 0, "bf16", False), (1024, 1, "bf16", False), (8192, 0, "bf16", False),
         (8192, 1, "bf16", False), (8192, 0, "mixed", False), (1024, 0, "bf16", True),
         (8192, 1, "mixed", True)]


@pytest.mark.parametrize("n_cap,bf16_scores,kv_fmt,prefill", CASES,
                         ids=[f"ncap{n}_{'bf16' if s else 'fp32'}_scores_{f}_kv"
                              f"{'_prefill' if pf else ''}" for n, s, f, pf in CASES])
def test_decode_step_over_the_state_cache(n_cap, bf16_scores, kv_fmt, prefill):
    """With `prefill`, request 1's first tokens are handed over from a prefill chunk; the
    oracle still takes every token one at a time (its decode equals a whole prefill)."""
    st = Stream(n_cap)
    ora = oracle_caches(st, kv_fmt)
    got = run_gpu(st, bf16_scores, kv_fmt, prefill)
    off = check_pages(st, ora, got, kv_fmt)
    check_selection_and_output(st, ora, got, off, bf16_scores)


# ---------------------------------------------------------------------------
# HCA: m' = 128, one entry per page, dense attention over every visible entry
# ---------------------------------------------------------------------------

HCA_M, HCA_N_TOK, HCA_N_CAP = 128, (2000, 900, 4100), 64


class HcaStream:
    def __init__(self, seed=2027):
        self.B = len(HCA_N_TOK)
        self.kv = W.make_state_stream(B=self.B, n_tok=max(HCA_N_TOK), m=HCA_M, c=C, overlap=0,
                                      io="bf16", seed=seed)
        g = np.random.default_rng(seed + 1)
        self.q = W.f32_to_bf16_bits(g.standard_normal((self.B, 1, H, C), np.float32))
        self.sink = g.standard_normal((H,), np.float32)
        self.pos = np.array([[t - 1] for t in HCA_N_TOK], np.int64)
        used = [t // HCA_M for t in HCA_N_TOK]
        self.n_pages = sum(used) + 3
        perm = g.permutation(self.n_pages).astype(np.int32)
        self.table = np.full((self.B, HCA_N_CAP), -1, np.int32)
        k = 0
        for b, u in enumerate(used):
            self.table[b, :u] = perm[k:k + u]
            k += u


@pytest.mark.parametrize("kv_fmt", ["bf16", "mixed"])
def test_hca_decode_step_over_the_state_cache(kv_fmt):
    import torch
    import long_context_sparse_08_b200 as csa

    st = HcaStream()
    mixed = kv_fmt == "mixed"
    B = st.B
    p = csa.make_params(m=HCA_M, overlap=0, c=C, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                        n_heads=H, n_win=N_WIN)
    torch.cuda.synchronize()
    csa.device_error()
    pages = torch.zeros((st.n_pages, 1, C + R), dtype=torch.uint8, device="cuda") if mixed \
        else torch.zeros((st.n_pages, 1, C), dtype=torch.int16, device="cuda")
    scales = torch.zeros((st.n_pages, 1), dtype=torch.float32, device="cuda") if mixed else None
    fmt = csa.CSA_MIXED_FP8_BF16 if mixed else csa.CSA_BF16
    state = torch.zeros((B, HCA_M, 2, C), dtype=torch.int16, device="cuda")
    ring = torch.zeros((B, N_WIN, C), dtype=torch.int16, device="cuda")
    src = {k: _up(st.kv[k]) for k in st.kv}
    for b, n in enumerate(HCA_N_TOK):
        pos_all = torch.zeros((n, 2), dtype=torch.int64, device="cuda")
        pos_all[:, 0] = torch.arange(n, device="cuda")
        tb = _up(st.table[b:b + 1])
        for t in range(n):
            csa.csa_state_append(p, csa.CSA_BF16, 1, pos_all[t, :1], src["Ca"][b, t:t + 1], None,
                                 src["Za"][b, t:t + 1], None, src["win"][b, t:t + 1],
                                 src["bias"], None, 1, state[b:b + 1], ring[b:b + 1],
                                 fmt, pages, scales, st.n_pages, 1, tb, HCA_N_CAP)
    torch.cuda.synchronize()
    assert csa.device_error() == 0, "appends"
    table = _up(st.table)
    kv = csa.paged_kv(fmt, pages, scales, table, st.n_pages, 1, HCA_N_CAP)
    need = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, B, 1, HCA_N_CAP)
    ws = torch.empty((max(need, 1),), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, 1, H, C), dtype=torch.int16, device="cuda")
    csa.hca_dense_mqa_paged(p, B, 1, _up(st.q), _up(st.pos), kv, ring, N_WIN, None,
                            _up(st.sink), None, out, ws, need)
    torch.cuda.synchronize()
    assert csa.device_error() == 0, "attention"
    got_pages = pages.cpu().numpy()
    got_pages = got_pages if mixed else got_pages.view(np.uint16)
    got_scales = scales.cpu().numpy() if mixed else None
    got = O.dec_bf16(out.cpu().numpy().view(np.uint16))
    for b, n in enumerate(HCA_N_TOK):
        pool = SC.PagePool(n // HCA_M + 1, 1, C)
        cs = SC.HcaState(pool, m=HCA_M, c=C, bias=O.dec_bf16(st.kv["bias"]), n_win=N_WIN, r=R,
                         base=BASE, eps=EPS, block_tokens=HCA_M)
        r = {k: O.dec_bf16(st.kv[k][b, :n]) for k in ("Ca", "Za", "win")}
        for t in range(n):
            cs.append(r["Ca"][t], r["Za"][t], r["win"][t])
        ent = cs.entries()
        pg = st.table[b, :len(ent)]
        check_kv_rows(got_pages[pg, 0], None if got_scales is None else got_scales[pg, 0], ent,
                      kv_fmt, f"HCA request {b}: entries")
        t = int(st.pos[b, 0])
        want = O.hca_query(O.dec_bf16(st.q[b, 0]), t, stored_kv(ent, kv_fmt),
                           O.visible_entries(t, HCA_M, HCA_N_CAP), r["win"], 0, st.sink, r=R,
                           base=BASE, eps=EPS, scale=1.0 / math.sqrt(C), n_win=N_WIN)
        U.check_out(got[b, 0], want, "bf16", f"HCA request {b}: output")
