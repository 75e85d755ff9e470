"""Pins of the oracle steps for the extensions beyond the decode path: BF16 index scores
into the selector, the mixed-precision KV entry, the grouped output projection and the
decode-time state cache.

As in test_oracle_pins, each test checks the oracle against something other than
itself: a library routine (torch's bf16 / e4m3 conversions, scipy's block-diagonal
matrix), a closed form, an order-free characterisation of a selection, an independent
whole-sequence computation, or the block sizes the pages print.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import csa_oracle as O
from oracle import state_cache as SC
from long_context_sparse_08_b200 import workloads as W

RNG = np.random.default_rng(4321)


# ---------------------------------------------------------------------------
# BF16 index scores  [【论文解读】DeepSeek-V4 二(四); DeepseekV4论文解析 三、实验]
# ---------------------------------------------------------------------------


def _torch_bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().double().numpy()


def test_round_to_bf16_matches_torch():
    g = np.random.default_rng(7)
    x = (g.standard_normal(20000) * np.exp2(g.integers(-140, 60, 20000))).astype(np.float32)
    # exact midpoints between neighbouring bf16 values, both parities of the lower one
    base = _torch_bf16(g.standard_normal(4000).astype(np.float32))
    ulp = np.exp2(np.floor(np.log2(np.abs(base))) - 7)
    mids = (base + 0.5 * ulp * np.sign(base)).astype(np.float32)
    assert np.all(mids.astype(np.float64) == base + 0.5 * ulp * np.sign(base))  # fp32-exact
    x = np.concatenate([x, mids, [0.0, -0.0]]).astype(np.float32)
    assert np.array_equal(O.round_to_bf16(x.astype(np.float64)), _torch_bf16(x))


def test_round_to_bf16_closed_forms():
    cases = {
        1 + 2 ** -8: 1.0,                  # half an ulp above 1: tie, 1 is even
        1 + 3 * 2 ** -8: 1 + 2 ** -6,      # tie between 1+2^-7 (odd) and 1+2^-6 (even)
        1 + 2 ** -8 + 2 ** -20: 1 + 2 ** -7,  # just past the tie
        2 - 2 ** -9: 2.0,                  # rounds up into the next binade
        -(3 + 2 ** -7): -3.0,              # [2, 4): ulp 2^-6, below half
        2.0 ** -130: 2.0 ** -130,          # subnormal multiple of 2^-133
        0.0: 0.0,
    }
    got = O.round_to_bf16(np.array(list(cases), np.float64))
    assert np.array_equal(got, np.array(list(cases.values())))


def test_bf16_selection_equals_exact_selection_on_bf16_scores():
    # scores that are bf16 values already (with many equal values) select as before
    s = _torch_bf16(RNG.standard_normal(5000).astype(np.float32) * 0.25)
    for k in (1, 37, 512, 5000, 6000):
        assert np.array_equal(O.topk_select_bf16(s, k), O.topk_select(s, k))


@pytest.mark.parametrize("n,k", [(3000, 100), (700, 64), (50, 80)])
def test_bf16_selection_characterisation(n, k):
    """Order-free description of the result: with R the scores rounded to bf16 (torch)
    and R_k the rounded value at the last selected slot, (a) every index with R > R_k is
    selected, (b) of the indices with R == R_k exactly the smallest are selected, (c) the
    list runs by (R desc, index asc), (d) slots past the candidates hold -1, and (e) any
    difference from the unrounded selection lies among indices rounding to R_k."""
    g = np.random.default_rng(n + k)
    s = g.standard_normal(n) * 3.0  # ~8 bit significands give many rounding ties
    R = _torch_bf16(s.astype(np.float32))
    sel = O.topk_select_bf16(s, k)
    kk = min(k, n)
    assert np.all(sel[kk:] == -1) and np.all(sel[:kk] >= 0)
    chosen = sel[:kk]
    assert len(set(chosen.tolist())) == kk
    Rk = R[chosen[-1]]
    assert set(np.flatnonzero(R > Rk)) <= set(chosen.tolist())
    tied = np.flatnonzero(R == Rk)
    n_tied_sel = int(np.sum(R[chosen] == Rk))
    assert sorted(chosen[R[chosen] == Rk].tolist()) == tied[:n_tied_sel].tolist()
    for a, b in zip(chosen[:-1], chosen[1:]):
        assert R[a] > R[b] or (R[a] == R[b] and a < b)
    exact = set(O.topk_select(s, k)[:kk].tolist())
    for i in exact.symmetric_difference(chosen.tolist()):
        assert R[i] == Rk


# ---------------------------------------------------------------------------
# mixed-precision KV entries  [【论文解读】DeepSeek-V4 一(三)4 item 1]
# ---------------------------------------------------------------------------


def test_mixed_kv_decoder_against_torch_formats():
    g = np.random.default_rng(11)
    codes = g.integers(0, 256, size=(6, 448), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    scale = np.exp2(g.integers(-6, 6, size=6)).astype(np.float32) * np.float32(1.25)
    rope = W.f32_to_bf16_bits(g.standard_normal((6, 64)).astype(np.float32))
    want_nope = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    want_nope = want_nope * scale.astype(np.float64)[:, None]
    want_rope = torch.from_numpy(rope.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = O.dec_mixed_kv(codes, scale, rope)
    assert got.shape == (6, 512)
    assert np.array_equal(got[:, :448], want_nope)
    assert np.array_equal(got[:, 448:], want_rope)


def test_mixed_kv_exact_rows_roundtrip():
    # rows whose first 448 dims are e4m3 values times a power of two with amax 448 * 2^e,
    # and whose last 64 dims are bf16 values, come back exactly (order and scale pinned)
    g = np.random.default_rng(12)
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    e = g.integers(-8, 8, size=4)
    nope = g.choice(grid, size=(4, 448)) * np.where(g.random((4, 448)) < 0.5, -1, 1)
    nope[:, 0] = 448.0
    nope = nope * np.exp2(e)[:, None]
    rope = _torch_bf16(g.standard_normal((4, 64)).astype(np.float32))
    x = np.concatenate([nope, rope], axis=1)
    codes, scale, bits = W.quant_mixed_kv(x.astype(np.float32), 64)
    assert np.array_equal(scale.astype(np.float64), np.exp2(e))
    assert np.array_equal(O.dec_mixed_kv(codes, scale, bits), x)


def test_mixed_kv_error_bound():
    g = np.random.default_rng(13)
    x = g.standard_normal((64, 512)).astype(np.float32)
    codes, scale, bits = W.quant_mixed_kv(x, 64)
    y = O.dec_mixed_kv(codes, scale, bits)
    xd = x.astype(np.float64)
    # bf16 RoPE dims: half an ulp; an ulp is at most 2^-7 of |x| (8 significant bits)
    assert np.all(np.abs(y[:, 448:] - xd[:, 448:]) <= np.abs(xd[:, 448:]) * 2.0 ** -8)
    # FP8 dims: half an e4m3 ulp (at most 2^-4 of |x|: 4 significant bits) for normals,
    # half the subnormal spacing 2^-9 (times the scale) below 2^-6
    s = scale.astype(np.float64)[:, None]
    bound = np.maximum(np.abs(xd[:, :448]) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(y[:, :448] - xd[:, :448]) <= bound)


# ---------------------------------------------------------------------------
# grouped output projection  [【论文解读】DeepSeek-V4 一(三)1(4), 2(2)]
# ---------------------------------------------------------------------------


def test_grouped_projection_routes_each_head_through_its_group():
    H, c, g, d_g, d = 8, 4, 2, 3, 5
    hg = H // g
    o = RNG.standard_normal((H, c))
    for a in range(H):
        for b in range(c):
            for j, k in ((0, 4), (2, 1)):
                w_grp = np.zeros((g, c * hg, d_g))
                w_out = np.zeros((g * d_g, d))
                w_grp[a // hg, (a % hg) * c + b, j] = 1.0
                w_out[(a // hg) * d_g + j, k] = 1.0
                want = np.zeros(d)
                want[k] = o[a, b]
                assert np.array_equal(O.grouped_output_projection(o, w_grp, w_out), want)


def test_one_group_per_head_with_identity_weights_is_the_concatenation():
    H, c = 6, 8
    o = RNG.standard_normal((H, c))
    w_grp = np.stack([np.eye(c)] * H)
    assert np.array_equal(O.grouped_output_projection(o, w_grp, np.eye(H * c)),
                          o.reshape(H * c))


@pytest.mark.parametrize("H,c,g,d_g,d", [(8, 16, 2, 24, 20), (16, 8, 16, 4, 7), (12, 4, 3, 10, 9)])
def test_grouped_projection_is_one_block_diagonal_projection(H, c, g, d_g, d):
    """The two projections compose into one of the flattened heads by the matrix
    blockdiag(W_1, ..., W_g) . W_out."""
    o = RNG.standard_normal((H, c))
    w_grp = RNG.standard_normal((g, c * H // g, d_g))
    w_out = RNG.standard_normal((g * d_g, d))
    dense = scipy.linalg.block_diag(*w_grp) @ w_out
    want = o.reshape(H * c) @ dense
    got = O.grouped_output_projection(o, w_grp, w_out)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_grouped_projection_shapes_of_the_model_table():
    # 三、预训练 (二) 模型配置: Flash n_h 64, g 8, d_g 1024, d 4096; Pro n_h 128, g 16,
    # d_g 1024, d 7168; c = 512. A group of n_h/g heads is c*n_h/g wide and d_g is smaller.
    for H, g, d_g in ((64, 8, 1024), (128, 16, 1024)):
        width = 512 * H // g
        assert width == 4096 and d_g < width


# ---------------------------------------------------------------------------
# state cache  [【论文解读】DeepSeek-V4 二(六); DeepseekV4论文解析 2. 从注意力公式到可部署系统]
# ---------------------------------------------------------------------------

CFG = dict(r=8, base=10000.0, eps=1e-6)


def _seq(n, c):
    g = np.random.default_rng(n * 31 + c)
    return [g.standard_normal((n, c)) for _ in range(5)]  # Ca, Cb, Za, Zb, window rows


def _whole_csa(Ca, Cb, Za, Zb, bias, m, n):
    nb = n // m
    ent = O.compress_csa(Ca[:m * nb], Cb[:m * nb], Za[:m * nb], Zb[:m * nb], bias, m)
    return O.finalize_entries(ent, 0, m, CFG["r"], CFG["base"], CFG["eps"])


def test_block_size_of_the_pages():
    # DeepseekV4论文解析 prints lcm(4, 128) = 128 raw tokens = 32 CSA entries = 1 HCA entry
    t = SC.block_tokens(4, 128)
    assert (t, t // 4, t // 128) == (128, 32, 1)


def test_csa_state_token_by_token_equals_whole_prefill():
    m, c, n, n_win = 4, 16, 2 * 128 + 37, 8
    Ca, Cb, Za, Zb, Wr = _seq(n, c)
    bias = RNG.standard_normal((2 * m, c))
    pool = SC.PagePool(8, 32, c, order=[5, 2, 7, 0, 3, 1, 6, 4])
    st = SC.CsaState(pool, m=m, c=c, bias=bias, n_win=n_win, **CFG)
    for t in range(n):
        done = st.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
        assert done == (t // m if (t + 1) % m == 0 else None)
        assert st.n_entries == (t + 1) // m
        if (t + 1) % (3 * m) == 0 or t == n - 1:
            want = _whole_csa(Ca, Cb, Za, Zb, bias, m, t + 1)
            got = st.entries()
            assert got.shape == want.shape
            assert np.allclose(got, want, rtol=0, atol=1e-13)


def test_hca_state_token_by_token_equals_whole_prefill():
    m, c, n, n_win = 16, 16, 16 * 5 + 3, 4
    C, _, Z, _, Wr = _seq(n, c)
    bias = RNG.standard_normal((m, c))
    pool = SC.PagePool(6, 1, c, order=[3, 0, 5, 1, 4, 2])
    st = SC.HcaState(pool, m=m, c=c, bias=bias, n_win=n_win, block_tokens=16, **CFG)
    for t in range(n):
        st.append(C[t], Z[t], Wr[t])
        assert st.held_rows() == (t + 1) % m
    nb = n // m
    want = O.finalize_entries(O.compress_hca(C[:m * nb], Z[:m * nb], bias, m), 0, m,
                              CFG["r"], CFG["base"], CFG["eps"])
    assert np.allclose(st.entries(), want, rtol=0, atol=1e-13)
    assert len(st.page_table) == nb


@pytest.mark.parametrize("n0", [0, 3, 64, 66, 130])
def test_prefill_then_decode_equals_whole_prefill(n0):
    m, c, n, n_win = 4, 16, 150, 8
    Ca, Cb, Za, Zb, Wr = _seq(n, c)
    bias = RNG.standard_normal((2 * m, c))
    st = SC.CsaState(SC.PagePool(4, 32, c), m=m, c=c, bias=bias, n_win=n_win, **CFG)
    st.resume(Ca[:n0], Cb[:n0], Za[:n0], Zb[:n0], _whole_csa(Ca, Cb, Za, Zb, bias, m, n0),
              Wr[:n0])
    for t in range(n0, n):
        st.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
        lo = max(t - n_win + 1, 0)
        assert np.array_equal(st.window_rows(t), Wr[lo:t + 1])
    assert np.allclose(st.entries(), _whole_csa(Ca, Cb, Za, Zb, bias, m, n), rtol=0, atol=1e-13)


@pytest.mark.parametrize("n0", [0, 5, 32, 47])
def test_hca_prefill_then_decode_equals_whole_prefill(n0):
    m, c, n, n_win = 16, 16, 16 * 4 + 7, 4
    C, _, Z, _, Wr = _seq(n, c)
    bias = RNG.standard_normal((m, c))
    whole = lambda k: O.finalize_entries(  # noqa: E731
        O.compress_hca(C[:m * (k // m)], Z[:m * (k // m)], bias, m), 0, m, CFG["r"],
        CFG["base"], CFG["eps"])
    st = SC.HcaState(SC.PagePool(8, 1, c), m=m, c=c, bias=bias, n_win=n_win, block_tokens=16,
                     **CFG)
    st.resume(C[:n0], Z[:n0], whole(n0), Wr[:n0])
    for t in range(n0, n):
        st.append(C[t], Z[t], Wr[t])
        assert np.array_equal(st.window_rows(t), Wr[max(t - n_win + 1, 0):t + 1])
    assert np.allclose(st.entries(), whole(n), rtol=0, atol=1e-13)


def test_indexer_key_state_gives_the_raw_compressed_keys():
    # keys take no RMSNorm / RoPE: token-by-token entries equal the plain compression
    m, c, n = 4, 16, 70
    Ca, Cb, Za, Zb, Wr = _seq(n, c)
    bias = RNG.standard_normal((2 * m, c))
    st = SC.CsaState(SC.PagePool(2, 32, c), m=m, c=c, bias=bias, n_win=4, finalize=False, **CFG)
    for t in range(n):
        st.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
    nb = n // m
    want = O.compress_csa(Ca[:m * nb], Cb[:m * nb], Za[:m * nb], Zb[:m * nb], bias, m)
    assert np.allclose(st.entries(), want, rtol=0, atol=1e-13)


def test_window_ring_holds_the_most_recent_rows():
    m, c, n_win = 4, 8, 6
    Ca, Cb, Za, Zb, Wr = _seq(40, c)
    st = SC.CsaState(SC.PagePool(2, 32, c), m=m, c=c, bias=np.zeros((2 * m, c)),
                     n_win=n_win, **CFG)
    for t in range(40):
        st.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
        w = st.window_rows(t)
        assert w.shape[0] == min(t + 1, n_win)
        assert np.array_equal(w, Wr[max(t - n_win + 1, 0):t + 1])


def test_pages_follow_blocks_and_are_reused_after_release():
    m, c = 4, 8
    Ca, Cb, Za, Zb, Wr = _seq(300, c)
    bias = RNG.standard_normal((2 * m, c))
    pool = SC.PagePool(3, 32, c, order=[2, 0, 1])
    a = SC.CsaState(pool, m=m, c=c, bias=bias, n_win=4, **CFG)
    for t in range(300):
        a.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
        # a page per started block of 128 raw tokens; the state itself stays bounded
        assert len(a.page_table) == math.ceil(((t + 1) // m) / 32)
        assert a.held_rows() <= 2 * m - 1
    assert a.page_table == [2, 0, 1]
    snap = a.entries().copy()
    a.release()
    assert sorted(pool.free) == [0, 1, 2]
    b = SC.CsaState(pool, m=m, c=c, bias=bias, n_win=4, **CFG)
    for t in range(300):  # the same tokens through reused pages give the same entries
        b.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
    assert np.array_equal(b.entries(), snap)


def test_finished_entries_are_never_rewritten():
    m, c = 4, 8
    Ca, Cb, Za, Zb, Wr = _seq(96, c)
    st = SC.CsaState(SC.PagePool(1, 32, c), m=m, c=c, bias=RNG.standard_normal((2 * m, c)),
                     n_win=4, **CFG)
    for t in range(41):
        st.append(Ca[t], Cb[t], Za[t], Zb[t], Wr[t])
    snap = st.entries().copy()
    for t in range(41, 96):  # later tokens, including a wildly different one
        st.append(Ca[t] * 1e3, Cb[t], Za[t] + 50, Zb[t], Wr[t])
    assert np.array_equal(st.entries()[:snap.shape[0]], snap)
