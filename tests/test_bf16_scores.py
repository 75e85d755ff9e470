"""BF16 index scores into the top-k selector (csa_index_topk_bf16; FP8, bf16 and MXFP4 keys)
against the oracle.

The scores are computed in fp32 and rounded once to bf16; the selector orders the bf16
values by (value desc, index asc). Checks:
  - every stored score is within one bf16 rounding of the oracle's score (plus the fp32
    tolerance of the scores);
  - the selection is valid for the scores the GPU stored (an order-free description: every
    larger value selected, the smallest indices among the values equal to the last one,
    the list ordered, -1 past the visible count);
  - it differs from the oracle's own BF16 selection only at near-ties of the k-th value;
  - its recall of the oracle's exact (unrounded) top-k equals that of the oracle's own BF16
    selection up to the near-tie swaps, and averages >= 0.99 over a case's queries (the
    pages report 99.7% for their data; the full-size Flash decode gives about 99.2% on the
    synthetic N(0,1) scores, 98.4-99.6% per query).
"""
import ctypes

import numpy as np
import pytest

import long_context_sparse_08_b200 as csa
from long_context_sparse_08_b200 import runner as R
from oracle import csa_oracle as O
from oracle import pipeline as P
import tests.parity_util as U

CASES = ["edge_decode_fp8_tc", "edge_decode_bf16_tc", "flash_decode_131k", "mid_prefill_bf16_tc",
         "edge_decode_mxfp4", "mid_decode_mxfp4", "mid_decode_mxfp4_sel"]


def test_checks_on_the_host():
    L = csa.lib()
    F = 0x10000
    p = csa.make_params(topk=512)
    need = csa.workspace_size(p, csa.CSA_WS_INDEX_TOPK_BF16, csa.CSA_BF16, 2, 1, 4096)
    full = csa.workspace_size(p, csa.CSA_WS_INDEX_TOPK, csa.CSA_BF16, 2, 1, 4096)
    assert need >= 2 * 4096 * 2 and need < full  # half the score bytes
    # f32 keys do not come from the tensor-core indexer
    s = L.csa_index_topk_bf16(ctypes.byref(p), csa.CSA_F32, 2, 1, 4096, F, None, F, F, None, F,
                              F, None, F, need, None)
    assert s == csa.CSA_ERR_UNSUPPORTED
    # N_cap not a multiple of 128
    s = L.csa_index_topk_bf16(ctypes.byref(p), csa.CSA_BF16, 2, 1, 4000, F, None, F, F, None, F,
                              F, None, F, need, None)
    assert s == csa.CSA_ERR_UNSUPPORTED
    s = L.csa_index_topk_bf16(ctypes.byref(p), csa.CSA_BF16, 2, 1, 4096, F, None, F, F, None, F,
                              None, None, F, need, None)
    assert s == csa.CSA_ERR_INVALID_ARG  # no output list
    s = L.csa_index_topk_bf16(ctypes.byref(p), csa.CSA_BF16, 2, 1, 4096, F, None, F, F, None, F,
                              F, None, F, need - 1, None)
    assert s == csa.CSA_ERR_WORKSPACE


def _valid_selection(sel, R, k):
    n = R.size
    kk = min(k, n)
    assert np.all(sel[kk:] == -1) and np.all(sel[:kk] >= 0)
    chosen = sel[:kk]
    if kk == 0:
        return
    assert len(set(chosen.tolist())) == kk
    Rk = R[chosen[-1]]
    assert set(np.flatnonzero(R > Rk)) <= set(chosen.tolist())
    tied = np.flatnonzero(R == Rk)
    n_tied = int(np.sum(R[chosen] == Rk))
    assert sorted(chosen[R[chosen] == Rk].tolist()) == tied[:n_tied].tolist()
    for a, b in zip(chosen[:-1], chosen[1:]):
        assert R[a] > R[b] or (R[a] == R[b] and a < b)


@pytest.mark.gpu
@pytest.mark.parametrize("name", CASES)
def test_bf16_scores_and_selection(name):
    import torch

    s, inp = U.inputs(name)
    res = P.run(s, inp, want_scores=True)
    dev = R.upload(inp, s)
    p = R.params_for(s)
    kdt = csa.DTYPES[s.idx]
    B, T, N = s.B, s.T, s.n_cap
    need = csa.workspace_size(p, csa.CSA_WS_INDEX_TOPK_BF16, kdt, B, T, N)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    out_idx = torch.empty((B, T, s.topk), dtype=torch.int32, device="cuda")
    sc16 = torch.zeros((B, T, N), dtype=torch.int16, device="cuda")
    csa.csa_index_topk_bf16(p, kdt, B, T, N, dev["qI"], dev.get("qI_scale"), dev["w"], dev["KI"],
                            dev.get("KI_scale"), dev["q_pos"], out_idx, sc16, ws, need)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got16 = sc16.cpu().numpy().view(np.uint16)
    idx = out_idx.cpu().numpy()
    recalls = []
    for (b, ti), ref in res["scores"].items():
        n = ref.size
        g = O.dec_bf16(got16[b, ti, :n])
        R_o = O.round_to_bf16(ref)
        lim = U.bf16_ulp(ref) + U.score_limit(ref, res["scale"][(b, ti)])[0]
        assert np.all(np.abs(g - R_o) <= lim), f"{name} b={b} t={ti}: bf16 scores"
        _valid_selection(idx[b, ti], g, s.topk)
        kk = min(s.topk, n)
        if kk == 0:
            continue
        mine = set(idx[b, ti, :kk].tolist())
        theirs = O.topk_select_bf16(ref, s.topk)[:kk]
        tau = R_o[theirs[-1]]
        tol = U.bf16_ulp(np.array([tau]))[0] + 1e-4 * max(abs(tau), 1e-3 * np.abs(ref).max())
        swaps = mine.symmetric_difference(theirs.tolist())
        for i in swaps:
            assert abs(ref[i] - tau) <= tol, f"{name} b={b} t={ti}: {i} is not a near-tie"
        # recall of the exact (unrounded) top-k: the GPU's equals the oracle's own BF16
        # selection's up to the near-tie swaps, each of which moves it by at most 1/k
        exact = set(O.topk_select(ref, s.topk)[:kk].tolist())
        r_gpu, r_ora = len(mine & exact) / kk, len(set(theirs.tolist()) & exact) / kk
        assert r_gpu >= r_ora - len(swaps) / (2 * kk) - 1e-12, f"{name} b={b} t={ti}: recall"
        recalls.append(r_gpu)
    if recalls:
        print(f"[bf16 recall] {name}: mean {np.mean(recalls):.4f} min {np.min(recalls):.4f} "
              f"over {len(recalls)} queries")
        assert np.mean(recalls) >= 0.99, f"{name}: mean recall {np.mean(recalls):.4f}"
