"""The checks of tests/test_decode_over_state_cache.py, run on the CPU: fed results made by
the oracle itself (pages filled with the input encoders' bytes through the page tables,
scores, selection and outputs from the oracle's steps) they pass, and each planted mistake
(a swapped selection order, a wrong member, a scaled output, one wrong score, one flipped
KV bit, four changed key codes, wrong mixed-row scales) fails them.
"""
import copy
import math

import numpy as np
import pytest

from oracle import csa_oracle as O
from long_context_sparse_08_b200 import workloads as W
import tests.test_decode_over_state_cache as T


def _oracle_results(st, ora, bf16_scores, kv_fmt):
    """What a correct GPU run returns, made from the oracle's own results."""
    mixed = kv_fmt == "mixed"
    row = T.C + T.R if mixed else T.C
    kvp = np.zeros((st.n_kv_pages, T.KV_ROWS, row), np.uint8 if mixed else np.uint16)
    kvs = np.zeros((st.n_kv_pages, T.KV_ROWS), np.float32) if mixed else None
    kp = np.zeros((st.n_key_pages, T.KEY_ROWS, T.D_I // 2), np.uint8)
    kx = np.zeros((st.n_key_pages, T.KEY_ROWS, 4), np.uint8)
    scores = np.zeros((st.B, 1, st.n_cap))
    idx = np.full((st.B, 1, T.K), -1, np.int32)
    out = np.zeros((st.B, 1, T.H, T.C))
    qI = O.dec_mxfp4(st.qI, st.qI_scale)
    for b, n in enumerate(T.N_TOK):
        o, ne = ora[b], n // T.M
        x = o["kv_f64"].astype(np.float32)
        pg, sl = T.page_rows_of(st.kv_table, T.KV_ROWS, b, ne)
        if mixed:
            codes, sc, rope = W.quant_mixed_kv(x, T.R)
            kvp[pg, sl] = np.concatenate([codes, rope.view(np.uint8).reshape(ne, -1)], axis=1)
            kvs[pg, sl] = sc
        else:
            kvp[pg, sl] = W.f32_to_bf16_bits(x)
        pg, sl = T.page_rows_of(st.key_table, T.KEY_ROWS, b, ne)
        kp[pg, sl] = o["keys_packed"]
        for p in np.unique(pg):  # exponents in the blocked order, one block per page
            rows = np.flatnonzero(pg == p)
            ex = np.zeros((T.KEY_ROWS, 4), np.uint8)
            ex[sl[rows]] = o["keys_ex"][rows]
            kx[p] = W.block_key_scales(ex)
        nv = st.n_vis(b)
        ref = O.index_scores(qI[b, 0], st.w[b, 0], o["keys"], nv)
        f32 = ref.astype(np.float32).astype(np.float64)
        scores[b, 0, :nv] = O.round_to_bf16(f32) if bf16_scores else f32
        sel = O.topk_select_bf16(ref, T.K) if bf16_scores else O.topk_select(f32, T.K)
        idx[b, 0] = sel
        o_t = O.csa_query(O.dec_bf16(st.q[b, 0]), int(st.pos[b, 0]), o["kv"], sel, o["win"], 0,
                          st.sink, r=T.R, base=T.BASE, eps=T.EPS, scale=1.0 / math.sqrt(T.C),
                          n_win=T.N_WIN)
        out[b, 0] = O.dec_bf16(W.f32_to_bf16_bits(o_t.astype(np.float32)))
    return dict(kv_pages=kvp, kv_scales=kvs, key_pages=kp, key_ex=kx, idx=idx, scores=scores,
                out=out)


def _fails(fn) -> bool:
    try:
        fn()
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("n_cap,bf16_scores,kv_fmt", sorted({c[:3] for c in T.CASES}))
def test_the_oracle_passes_its_own_checks(n_cap, bf16_scores, kv_fmt):
    st = T.Stream(n_cap)
    ora = T.oracle_caches(st, kv_fmt)
    got = _oracle_results(st, ora, bf16_scores, kv_fmt)
    off = T.check_pages(st, ora, got, kv_fmt)
    assert all(len(x) == 0 for x in off)
    T.check_selection_and_output(st, ora, got, off, bf16_scores)


def test_planted_mistakes_fail_the_checks():
    st = T.Stream(1024)
    ora = T.oracle_caches(st, "bf16")
    got = _oracle_results(st, ora, 0, "bf16")
    off = T.check_pages(st, ora, got, "bf16")
    sel_out = lambda g: T.check_selection_and_output(st, ora, g, off, 0)  # noqa: E731

    g = copy.deepcopy(got)
    g["idx"][1, 0, [3, 4]] = g["idx"][1, 0, [4, 3]]
    assert _fails(lambda: sel_out(g)), "swapped order"
    g = copy.deepcopy(got)
    g["idx"][0, 0, -1] = np.setdiff1d(np.arange(st.n_vis(0)), g["idx"][0, 0])[-1]
    assert _fails(lambda: sel_out(g)), "wrong member"
    g = copy.deepcopy(got)
    g["out"][2] *= 1.03
    assert _fails(lambda: sel_out(g)), "scaled output"
    g = copy.deepcopy(got)
    g["scores"][0, 0, 5] += 0.5
    assert _fails(lambda: sel_out(g)), "one score"
    g = copy.deepcopy(got)
    g["kv_pages"][st.kv_table[1, 0], 3, 7] ^= 0x40
    assert _fails(lambda: T.check_pages(st, ora, g, "bf16")), "one KV bit"
    g = copy.deepcopy(got)
    for page, slot in ((1, 3), (1, 9), (0, 9), (0, 19)):
        g["key_pages"][st.key_table[0, page], slot, 2] ^= 0x11
    assert _fails(lambda: T.check_pages(st, ora, g, "bf16")), "four key codes"

    ora_m = T.oracle_caches(st, "mixed")
    got_m = _oracle_results(st, ora_m, 0, "mixed")
    g = copy.deepcopy(got_m)
    g["kv_scales"] = g["kv_scales"] * 1.2
    assert _fails(lambda: T.check_pages(st, ora_m, g, "mixed")), "mixed-row scales"
