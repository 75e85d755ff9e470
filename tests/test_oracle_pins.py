"""Pins of the float64 oracle against what the pages and the mathematics fix.

Every test here checks the oracle against something other than itself: a closed
form, an invariant, a special case that reduces to a library routine, a brute force
written independently, or the counts the pages print. Each is chosen so that a
plausible slip in the oracle (a dropped branch, a wrong block offset, a sign, a
transposed operand, a wrong frequency) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from oracle import pipeline as P
from long_context_sparse_08_b200 import workloads as W

RNG = np.random.default_rng(1234)


def _rand(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------------------
# stored formats
# ---------------------------------------------------------------------------

def test_bf16_decoder_matches_torch():
    x = torch.randn(4096, dtype=torch.float32).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.dec_bf16(bits), x.double().numpy())


def test_e4m3_decoder_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.dec_e4m3(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and nan.sum() == 2  # 0x7F and 0xFF
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e2m1_decoder_is_the_ocp_table():
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    got = O.dec_e2m1(np.arange(16))
    np.testing.assert_array_equal(got[:8], table)
    np.testing.assert_array_equal(got[8:], [-v for v in table])


def test_mxfp4_exact_grid_roundtrip_and_nibble_order():
    # a block whose values sit on the e2m1 grid times 2^e decodes exactly
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    x = np.concatenate([grid, -grid, grid[::-1], -grid[::-1]]).astype(np.float32) * 2.0 ** -3
    packed, sc = W.quant_mxfp4(x[None])
    assert sc[0, 0] == 127 - 3 + 0  # amax 6*2^-3 -> floor(log2)=-1 -> E=-3
    np.testing.assert_array_equal(O.dec_mxfp4(packed, sc)[0], x.astype(np.float64))
    # element 0 lives in the low nibble of byte 0, element 1 in the high nibble
    assert packed[0, 0] & 0xF == 0 and packed[0, 0] >> 4 == 1


def test_mxfp4_error_bound():
    x = RNG.standard_normal((64, 128)).astype(np.float32)
    packed, sc = W.quant_mxfp4(x)
    d = O.dec_mxfp4(packed, sc)
    unit = np.repeat(O.dec_e8m0(sc), 32, axis=-1)
    # amax/2^E lies in [4, 8): values in (6, 8)*2^E saturate to 6*2^E (error < 2*2^E);
    # below 6*2^E the grid spacing is at most 2*2^E (error <= 2^E)
    err = np.abs(d - x)
    assert np.all(err < 2.0 * unit)
    inside = np.abs(x) <= 6 * unit
    assert np.all(err[inside] <= unit[inside] + 1e-12)


def test_blocked_key_scale_layout():
    nat = RNG.integers(0, 255, size=(2, 256, 4)).astype(np.uint8)
    blk = W.block_key_scales(nat)
    np.testing.assert_array_equal(O.unblock_key_scales(blk), nat)
    # explicit position of one key's scales: key 32*j + i of block 1 at word 4*i + j
    i, j = 5, 3
    flat = blk[0].reshape(-1)
    np.testing.assert_array_equal(flat[512 + 16 * i + 4 * j: 512 + 16 * i + 4 * j + 4],
                                  nat[0, 128 + 32 * j + i])


def test_fp8_rowwise_error_bound():
    x = RNG.standard_normal((32, 128)).astype(np.float32)
    codes, sc = W.quant_fp8_rowwise(x)
    d = O.dec_fp8_rows(codes, sc)
    assert np.all(np.abs(d - x) <= np.abs(x) * 2.0 ** -4 + sc[:, None] * 2.0 ** -9 + 1e-12)
    assert np.allclose(np.abs(d).max(axis=1), 448.0 * sc, rtol=1e-6)


# ---------------------------------------------------------------------------
# compression (overlapped CSA and non-overlapped HCA)
# ---------------------------------------------------------------------------

def _csa_inputs(n=32, c=6, m=4):
    return _rand(n, c), _rand(n, c), _rand(n, c), _rand(n, c), 0.3 * _rand(2 * m, c)


def test_pool_weights_sum_to_one_and_first_block_has_no_b_branch():
    Ca, Cb, Za, Zb, bias = _csa_inputs()
    m = 4
    for i in range(8):
        S = O.csa_pool_weights(Za, Zb, bias[:m], bias[m:], m, i)
        assert S.shape == (2 * m, 6)
        assert np.all(np.abs(S.sum(axis=0) - 1.0) < 1e-12)
        assert np.all(S >= 0)
        if i == 0:
            assert np.all(S[m:] == 0.0)


def test_constant_logits_give_plain_mean():
    Ca, Cb, Za, Zb, bias = _csa_inputs()
    m = 4
    Z = np.full_like(Za, 0.7)
    out = O.compress_csa(Ca, Cb, Z, Z, np.zeros_like(bias), m)
    np.testing.assert_allclose(out[0], Ca[0:4].mean(axis=0), rtol=0, atol=1e-13)
    for i in range(1, 8):
        ref = np.concatenate([Ca[4 * i:4 * i + 4], Cb[4 * i - 4:4 * i]]).mean(axis=0)
        np.testing.assert_allclose(out[i], ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("branch", ["a", "b"])
def test_spike_logit_selects_that_token(branch):
    Ca, Cb, Za, Zb, bias = _csa_inputs()
    m = 4
    for (i, r, j) in [(1, 0, 0), (3, 2, 5), (7, 3, 2), (5, 1, 4)]:
        Za2, Zb2 = Za.copy(), Zb.copy()
        if branch == "a":
            Za2[m * i + r, j] += 60.0
            want = Ca[m * i + r, j]
        else:
            Zb2[m * (i - 1) + r, j] += 60.0
            want = Cb[m * (i - 1) + r, j]
        out = O.compress_csa(Ca, Cb, Za2, Zb2, bias, m)
        assert abs(out[i, j] - want) < 1e-12 * max(1.0, abs(want)) + 1e-20 + 1e-11
        # the other channels of that entry are untouched by the spike
        base = O.compress_csa(Ca, Cb, Za, Zb, bias, m)
        others = [k for k in range(6) if k != j]
        np.testing.assert_array_equal(out[i, others], base[i, others])


def test_bias_row_is_the_in_block_offset():
    Ca, Cb, _, _, _ = _csa_inputs()
    m = 4
    Z = np.zeros_like(Ca)
    for r in range(m):
        bias = np.zeros((2 * m, 6))
        bias[r, 2] = 60.0  # B^a row r
        out = O.compress_csa(Ca, Cb, Z, Z, bias, m)
        np.testing.assert_allclose(out[:, 2], Ca[r::m, 2], atol=1e-11)
        bias = np.zeros((2 * m, 6))
        bias[m + r, 3] = 60.0  # B^b row r
        out = O.compress_csa(Ca, Cb, Z, Z, bias, m)
        np.testing.assert_allclose(out[1:, 3], Cb[r::m, 3][:-1], atol=1e-11)
        # block 0 has no b-branch: its entry is the plain mean of the a-block
        np.testing.assert_allclose(out[0, 3], Ca[0:m, 3].mean(), atol=1e-13)


def test_m1_two_term_closed_form():
    # m = 1: each entry mixes two tokens with a logistic weight
    Ca, Cb, Za, Zb, bias = _csa_inputs(n=5, c=1, m=1)
    out = O.compress_csa(Ca, Cb, Za, Zb, bias, 1)
    assert out[0, 0] == pytest.approx(Ca[0, 0], abs=1e-15)
    for i in range(1, 5):
        la = Za[i, 0] + bias[0, 0]
        lb = Zb[i - 1, 0] + bias[1, 0]
        wa = 1.0 / (1.0 + math.exp(lb - la))
        assert out[i, 0] == pytest.approx(wa * Ca[i, 0] + (1 - wa) * Cb[i - 1, 0], abs=1e-14)


def test_compression_is_block_causal():
    Ca, Cb, Za, Zb, bias = _csa_inputs()
    m = 4
    base = O.compress_csa(Ca, Cb, Za, Zb, bias, m)
    for s in range(7):
        cut = m * (s + 1)
        pert = [x.copy() for x in (Ca, Cb, Za, Zb)]
        for x in pert:
            x[cut:] += _rand(*x[cut:].shape)
        out = O.compress_csa(*pert, bias, m)
        np.testing.assert_array_equal(out[:s + 1], base[:s + 1])
        assert np.all(out[s + 1] != base[s + 1])


def test_chunked_compression_with_tail_state_equals_whole():
    Ca, Cb, Za, Zb, bias = _csa_inputs(n=40)
    m = 4
    whole = O.compress_csa(Ca, Cb, Za, Zb, bias, m)
    cut = 16
    part2 = O.compress_csa(Ca[cut:], Cb[cut:], Za[cut:], Zb[cut:], bias, m,
                           prev_Cb=Cb[cut - m:cut], prev_Zb=Zb[cut - m:cut])
    np.testing.assert_allclose(part2, whole[cut // m:], rtol=0, atol=1e-14)


def test_hca_compression_closed_forms():
    m, c = 16, 5
    C, Z = _rand(64, c), _rand(64, c)
    bias = 0.1 * _rand(m, c)
    out = O.compress_hca(C, np.full_like(Z, -2.0), np.zeros_like(bias), m)
    np.testing.assert_allclose(out, C.reshape(4, m, c).mean(axis=1), atol=1e-13)
    Z2 = Z.copy()
    Z2[m * 2 + 7, 1] += 80.0
    out = O.compress_hca(C, Z2, bias, m)
    assert out[2, 1] == pytest.approx(C[m * 2 + 7, 1], abs=1e-12)
    # weights of each block and channel sum to 1: pooling a constant gives the constant
    out = O.compress_hca(np.full_like(C, 3.25), Z, bias, m)
    np.testing.assert_allclose(out, 3.25, atol=1e-13)


# ---------------------------------------------------------------------------
# RMSNorm and partial RoPE
# ---------------------------------------------------------------------------

def test_rms_norm_closed_forms():
    x = _rand(7, 64)
    eps = 1e-6
    y = O.rms_norm(x, eps)
    ms = np.mean(x * x, axis=1)
    np.testing.assert_allclose(np.mean(y * y, axis=1), ms / (ms + eps), rtol=1e-12)
    np.testing.assert_allclose(y / x, (1 / np.sqrt(ms + eps))[:, None] * np.ones_like(x),
                               rtol=1e-12)
    g = _rand(64)
    np.testing.assert_allclose(O.rms_norm(x, eps, g), y * g, rtol=1e-13)
    assert O.rms_norm(np.full((1, 4), -2.0), 0.0)[0, 0] == pytest.approx(-1.0, abs=1e-15)


def test_rope_closed_forms():
    c, r = 8, 4
    e = np.zeros(c)
    e[c - r] = 1.0  # first dim of pair p=0 of the rotated slice
    y = O.rope(e, 1, r, 10000.0)
    assert y[c - r] == pytest.approx(math.cos(1.0), abs=1e-15)
    assert y[c - r + 1] == pytest.approx(math.sin(1.0), abs=1e-15)
    e = np.zeros(c)
    e[c - 2] = 1.0  # pair p=1 turns at base^(-2/r) = 1e-2 rad per position
    y = O.rope(e, 100, r, 10000.0)
    assert y[c - 2] == pytest.approx(math.cos(1.0), abs=1e-12)
    assert y[c - 1] == pytest.approx(math.sin(1.0), abs=1e-12)
    x = _rand(5, c)
    z = O.rope(x, 37, r, 10000.0)
    np.testing.assert_array_equal(z[:, :c - r], x[:, :c - r])  # only the last r dims
    np.testing.assert_allclose(np.linalg.norm(z, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    np.testing.assert_allclose(O.rope(z, -37, r, 10000.0), x, atol=1e-14)


def test_rope_scores_depend_on_relative_position_only():
    c, r = 16, 8
    q, k = _rand(c), _rand(c)
    a = O.rope(q, 50, r, 10000.0) @ O.rope(k, 20, r, 10000.0)
    b = O.rope(q, 530, r, 10000.0) @ O.rope(k, 500, r, 10000.0)
    assert a == pytest.approx(b, rel=1e-12)


# ---------------------------------------------------------------------------
# indexer, visibility, top-k
# ---------------------------------------------------------------------------

def test_index_scores_brute_force_loops():
    H, d, N = 3, 5, 7
    q, K, w = _rand(H, d), _rand(N, d), _rand(H)
    got = O.index_scores(q, w, K, N)
    for s in range(N):
        tot = 0.0
        for h in range(H):
            dot = 0.0
            for j in range(d):
                dot += q[h][j] * K[s][j]
            tot += w[h] * (dot if dot > 0 else 0.0)
        assert got[s] == pytest.approx(tot, rel=1e-12, abs=1e-12)
    assert O.index_scores(q, w, K, 3).shape == (3,)


def test_index_scores_relu_drops_negative_heads():
    d = 4
    k = np.array([[1.0, 2.0, 0.0, -1.0]])
    q = np.array([[1.0, 0, 0, 0], [-1.0, 0, 0, 0], [0, 1.0, 0, 0]])  # dots 1, -1, 2
    w = np.array([2.0, 100.0, -0.5])
    assert O.index_scores(q, w, k, 1)[0] == pytest.approx(2.0 * 1 + 0 - 0.5 * 2)


def test_visibility_is_strict_block_causal():
    m = 4
    for s in range(10):
        assert O.visible_entries(m * (s + 1) - 1, m, 10 ** 9) == s  # block s incomplete
        assert O.visible_entries(m * (s + 1), m, 10 ** 9) == s + 1
    assert O.visible_entries(3, 4, 100) == 0
    assert O.visible_entries(10 ** 6, 4, 17) == 17


def test_counts_printed_by_the_pages(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "entry_counts.json")))
    t = g["ctx_tokens"]  # the decode query after a 1M-token context
    assert O.visible_entries(t, g["csa_m"], 10 ** 9) == g["csa_candidates"]
    nw = len(O.window_positions(t, g["n_win"], t - g["n_win"] + 1, g["n_win"]))
    assert nw == g["n_win"]
    assert g["pro_topk"] + nw == g["pro_core_entries"]
    assert g["flash_topk"] + nw == g["flash_core_entries"]
    assert O.visible_entries(t, g["hca_m"], 10 ** 9) == g["hca_entries"]
    assert nw == g["hca_window_entries"]
    blk = g["block_tokens"]
    assert math.lcm(g["csa_m"], g["hca_m"]) == blk
    assert O.visible_entries(blk, g["csa_m"], 10 ** 9) == g["csa_entries_per_block"]
    assert O.visible_entries(blk, g["hca_m"], 10 ** 9) == g["hca_entries_per_block"]


def test_topk_matches_sort_and_breaks_ties_by_index():
    s = RNG.standard_normal(200)
    got = O.topk_select(s, 20)
    ref = sorted(range(200), key=lambda i: (-s[i], i))[:20]
    assert list(got) == ref
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0, -1.0])
    assert list(O.topk_select(s, 4)) == [1, 2, 4, 3]
    assert list(O.topk_select(s[:2], 4)) == [1, 0, -1, -1]
    assert list(O.topk_select(np.zeros(0), 3)) == [-1, -1, -1]
    # the selected set is the argpartition set
    big = RNG.standard_normal(5000)
    assert set(O.topk_select(big, 64)) == set(np.argpartition(-big, 64)[:64])


# ---------------------------------------------------------------------------
# core attention with sink
# ---------------------------------------------------------------------------

def test_single_row_closed_forms():
    c = 8
    row = _rand(1, c)
    q = _rand(2, c)
    np.testing.assert_allclose(O.core_attention(q, row, None, 0.3), np.vstack([row, row]),
                               atol=1e-15)
    z = 0.3 * (q @ row[0])
    sink = np.array([0.5, -1.0])
    got = O.core_attention(q, row, sink, 0.3)
    for h in range(2):
        frac = math.exp(z[h]) / (math.exp(z[h]) + math.exp(sink[h]))
        np.testing.assert_allclose(got[h], frac * row[0], atol=1e-14)


def test_no_sink_is_plain_softmax_attention():
    q, rows = _rand(3, 16), _rand(11, 16)
    p = torch.softmax(torch.from_numpy(q @ rows.T * 0.25), dim=1).numpy()
    np.testing.assert_allclose(O.core_attention(q, rows, None, 0.25), p @ rows, atol=1e-14)


def test_sink_only_lowers_mass():
    q, rows = _rand(4, 16), _rand(9, 16)
    sink = _rand(4)
    o_s = O.core_attention(q, rows, sink, 0.25)
    o_n = O.core_attention(q, rows, None, 0.25)
    S = np.exp(q @ rows.T * 0.25).sum(axis=1)
    keep = S / (S + np.exp(sink))
    np.testing.assert_allclose(o_s, o_n * keep[:, None], rtol=1e-12, atol=1e-14)
    assert np.all((keep > 0) & (keep < 1))
    np.testing.assert_allclose(O.core_attention(q, rows, np.full(4, -np.inf), 0.25), o_n,
                               atol=1e-15)


def test_uniform_logits_give_scaled_mean():
    rows = _rand(6, 8)
    q = np.zeros((1, 8))
    got = O.core_attention(q, rows, np.array([0.0]), 1.0)
    np.testing.assert_allclose(got[0], rows.sum(axis=0) / 7.0, atol=1e-14)


# ---------------------------------------------------------------------------
# whole query: brute force, causality, shift invariance
# ---------------------------------------------------------------------------

def _tiny_problem(seed=7, n=64, c=16, r=8, m=4, Hq=3, HI=2, dI=8, shift=0):
    g = np.random.default_rng(seed)
    Ca, Cb, Za, Zb = (g.standard_normal((n, c)) for _ in range(4))
    bias = 0.1 * g.standard_normal((2 * m, c))
    q = g.standard_normal((n, Hq, c))
    qI = g.standard_normal((n, HI, dI))
    KI = g.standard_normal((n // m, dI))
    w = g.uniform(0, 1, (n, HI))
    raw_win = g.standard_normal((n, c))
    sink = g.standard_normal(Hq)
    comp = O.compress_csa(Ca, Cb, Za, Zb, bias, m)
    kv = O.finalize_entries(comp, shift // m, m, r, 10000.0, 1e-6)
    win = O.rope(O.rms_norm(raw_win, 1e-6), shift + np.arange(n), r, 10000.0)
    return dict(q=q, qI=qI, KI=KI, w=w, kv=kv, win=win, sink=sink, m=m, r=r, c=c)


def _csa_out(p, t, k, n_win, shift=0):
    n_vis = O.visible_entries(t, p["m"], p["kv"].shape[0])
    sc = O.index_scores(p["qI"][t], p["w"][t], p["KI"], n_vis)
    sel = O.topk_select(sc, k)
    return O.csa_query(p["q"][t], t + shift, p["kv"], sel, p["win"], shift, p["sink"],
                       r=p["r"], base=10000.0, eps=1e-6, scale=1 / math.sqrt(p["c"]),
                       n_win=n_win)


def test_full_coverage_equals_dense_attention():
    p = _tiny_problem()
    scale = 1 / math.sqrt(p["c"])
    for t in [0, 3, 4, 17, 40, 63]:
        got = _csa_out(p, t, k=64, n_win=64)
        # dense attention written separately: all visible entries and all tokens <= t
        n_vis = t // p["m"]
        keys = np.concatenate([p["kv"][:n_vis], p["win"][:t + 1]])
        qh = O.rope(O.rms_norm(p["q"][t], 1e-6), t, p["r"], 10000.0)
        logits = np.einsum("hc,lc->hl", qh, keys) * scale
        full = np.concatenate([logits, p["sink"][:, None]], axis=1)
        wts = np.exp(full - full.max(axis=1, keepdims=True))
        wts /= wts.sum(axis=1, keepdims=True)
        o = np.einsum("hl,lc->hc", wts[:, :-1], keys)
        o = O.rope(o, -t, p["r"], 10000.0)
        np.testing.assert_allclose(got, o, rtol=0, atol=1e-12)


def test_future_tokens_do_not_change_a_query():
    p = _tiny_problem()
    t = 29
    base = _csa_out(p, t, k=4, n_win=8)
    p2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
    n_vis = t // 4
    p2["kv"][n_vis:] += 1.0
    p2["KI"][n_vis:] += 1.0
    p2["win"][t + 1:] += 1.0
    p2["q"][t + 1:] += 1.0
    np.testing.assert_array_equal(_csa_out(p2, t, k=4, n_win=8), base)
    p2["win"][t] += 1.0  # the query's own token is in its window
    assert not np.array_equal(_csa_out(p2, t, k=4, n_win=8), base)


def test_output_is_invariant_to_a_global_position_shift():
    a = _tiny_problem(shift=0)
    b = _tiny_problem(shift=4 * 1000)
    for t in [15, 22, 63]:  # windows not clipped at position 0
        np.testing.assert_allclose(_csa_out(a, t, 6, 16, 0), _csa_out(b, t, 6, 16, 4000),
                                   rtol=0, atol=1e-11)


def test_window_positions_include_the_query():
    assert list(O.window_positions(0, 128, 0, 1)) == [0]
    assert list(O.window_positions(5, 3, 0, 10)) == [3, 4, 5]
    assert len(O.window_positions(1000, 128, 873, 128)) == 128


# ---------------------------------------------------------------------------
# the workload driver
# ---------------------------------------------------------------------------

def test_pipeline_tiny_first_queries_window_only():
    s = W.SHAPES["tiny_prefill_f32"]
    inp = W.make_inputs(s)
    res = P.run(s, inp, [(0, 0), (0, 3), (0, 4), (0, 255)])
    assert list(res["idx"][(0, 0)]) == [-1] * 16
    assert list(res["idx"][(0, 4)])[:2] == [0, -1]
    assert len(res["scores"][(0, 255)]) == 63
    # t = 0: one window row (the token itself) plus a zero sink
    qh = O.query_prep(inp["q"][0, 0], 0, 16, 1e4, 1e-6)
    row = inp["win_kv"][0, 0].astype(np.float64)
    z = qh @ row / 8.0
    frac = np.exp(z) / (np.exp(z) + 1.0)
    np.testing.assert_allclose(res["out"][(0, 0)], frac[:, None] * row[None], atol=1e-13)


def test_index_score_scale_bounds_the_score():
    H, d, N = 6, 8, 40
    q, K, w = _rand(H, d), _rand(N, d), _rand(H)
    I = O.index_scores(q, w, K, N)
    A = O.index_score_scale(q, w, K, N)
    assert np.all(A >= np.abs(I) - 1e-12)
    np.testing.assert_allclose(O.index_score_scale(q, np.abs(w), K, N),
                               O.index_scores(q, np.abs(w), K, N), rtol=1e-14)
