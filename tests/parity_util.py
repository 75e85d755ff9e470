"""Comparison rules between the CUDA path and the float64 oracle.

Tolerances (restated from the build's target):
  - compressed entries and indexer scores agree to 1e-4 relative in fp32. A score must
    meet |dI| <= 1e-4 * max(|I|, 1e-3 * max_s |I|) (the "1e-4 relative" rule with a floor
    at a thousandth of the row's largest score). The one exemption is a score that signed
    head weights cancel: where |I| < A / 8, with A = sum_h |w_h| ReLU(q_h . k) >= |I| the
    magnitude of the terms summed, fp32 rounding of the sum scales with A, not with |I|,
    and such a score must instead meet |dI| <= 1e-4 * A. Every exemption is counted;
  - a compressed row: ||d||/||ref|| <= 1e-4 and |d| <= 1e-4 rms(ref); a bf16 row is that
    fp32 bound plus one rounding to bf16 (half a bf16 ulp);
  - top-k sets are identical except at near-ties: with tau the oracle's k-th largest score
    and tol = 1e-4 * max(|tau|, 1e-3 max|I|), every entry with I > tau + tol is selected and
    every selected entry has I >= tau - tol;
  - bf16 outputs: relative RMS error <= 5e-3 and max abs error <= 2e-2 (fp32 outputs: 2e-5
    and 2e-4), against the oracle run on the same selection.
"""
from __future__ import annotations

import functools

import numpy as np

from long_context_sparse_08_b200 import workloads as W


@functools.lru_cache(maxsize=4)
def inputs(name: str):
    s = W.SHAPES[name]
    return s, W.make_inputs(s)


def dec_out(t, io: str) -> np.ndarray:
    import torch

    return t.float().cpu().numpy().astype(np.float64) if io == "bf16" else \
        t.cpu().numpy().astype(np.float64)


# counts of the score checks in this process: scores checked, scores that meet the plain
# relative rule, and cancellation exemptions (see the module docstring)
SCORE_STATS = {"checked": 0, "relative": 0, "cancelled": 0}


def score_limit(ref, scale):
    """Per-score bound of the module docstring's rule: 1e-4 * max(|I|, 1e-3 * max|I|), and
    for a cancelling score (|I| < A / 8) the larger of that and 1e-4 * A. Returns (bound,
    mask of the scores where only the cancellation exemption can hold)."""
    ref = np.asarray(ref, np.float64)
    scale = np.asarray(scale, np.float64)
    rel = 1e-4 * np.maximum(np.abs(ref), 1e-3 * np.abs(ref).max()) if ref.size else ref
    cancel = np.abs(ref) < scale / 8
    return np.where(cancel, np.maximum(rel, 1e-4 * scale), rel), cancel & (1e-4 * scale > rel)


def check_scores(gpu: np.ndarray, ref: np.ndarray, scale: np.ndarray, what=""):
    """Scores against the oracle under the rule of the module docstring. Returns
    (n, n exempted as cancelling, worst error / the plain relative bound) and adds the
    counts to SCORE_STATS."""
    ref = np.asarray(ref, np.float64)
    gpu = np.asarray(gpu, np.float64)
    scale = np.asarray(scale, np.float64)
    assert gpu.shape == ref.shape == scale.shape, what
    if ref.size == 0:
        return 0, 0, 0.0
    assert np.all(scale >= np.abs(ref) * (1 - 1e-12)), f"{what}: scale below |I|"
    err = np.abs(gpu - ref)
    rel = 1e-4 * np.maximum(np.abs(ref), 1e-3 * np.abs(ref).max())
    lim, _ = score_limit(ref, scale)
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} scores off; worst err/bound "
                           f"{(err / lim).max():.3e}")
    n_c = int((err > rel).sum())  # passed only through the cancellation exemption
    worst = float((err / rel).max())
    SCORE_STATS["checked"] += ref.size
    SCORE_STATS["relative"] += ref.size - n_c
    SCORE_STATS["cancelled"] += n_c
    print(f"[scores] {what}: n={ref.size} exempt(cancelling)={n_c} "
          f"worst err/(1e-4 max(|I|,floor))={worst:.2e}")
    return ref.size, n_c, worst


def check_topk(gpu_idx: np.ndarray, ref_scores: np.ndarray, k: int, gpu_scores=None, what=""):
    """Near-tie rule of the module docstring, plus structure: distinct valid indices first,
    -1 padding after, and (given the GPU's own scores) ordered by (score desc, index asc)."""
    ref = np.asarray(ref_scores, np.float64)
    n = ref.size
    nv = min(k, n)
    gi = np.asarray(gpu_idx, np.int64)
    assert np.all(gi[nv:] == -1), f"{what}: padding"
    sel = gi[:nv]
    assert np.all((sel >= 0) & (sel < n)), f"{what}: index out of range"
    assert np.unique(sel).size == nv, f"{what}: duplicate indices"
    if nv == 0:
        return 0
    if nv == n:
        return 0
    tau = np.sort(ref)[::-1][k - 1]
    tol = 1e-4 * max(abs(tau), 1e-3 * np.abs(ref).max())
    must = np.nonzero(ref > tau + tol)[0]
    missing = np.setdiff1d(must, sel)
    assert missing.size == 0, f"{what}: {missing.size} clearly-top entries missing"
    assert np.all(ref[sel] >= tau - tol), f"{what}: a selected entry is clearly below rank k"
    if gpu_scores is not None:
        gs = np.asarray(gpu_scores, np.float32)[sel]
        for j in range(nv - 1):
            a, b = gs[j], gs[j + 1]
            assert a > b or (a == b and sel[j] < sel[j + 1]), f"{what}: order at {j}"
    ref_set = set(np.argsort(-ref, kind="stable")[:k].tolist())
    return len(ref_set - set(sel.tolist()))


def recall(gpu_idx, ref_idx) -> float:
    g = set(int(i) for i in gpu_idx if i >= 0)
    r = set(int(i) for i in ref_idx if i >= 0)
    return 1.0 if not r else len(g & r) / len(r)


def check_out(gpu: np.ndarray, ref: np.ndarray, io: str, what=""):
    ref = np.asarray(ref, np.float64)
    d = np.asarray(gpu, np.float64) - ref
    rel_rms = np.sqrt((d * d).sum() / max((ref * ref).sum(), 1e-300))
    mx = np.abs(d).max() if d.size else 0.0
    lim_rms, lim_max = (5e-3, 2e-2) if io == "bf16" else (2e-5, 2e-4)
    assert rel_rms <= lim_rms and mx <= lim_max, \
        f"{what}: rel RMS {rel_rms:.3e} (<= {lim_rms}), max abs {mx:.3e} (<= {lim_max})"
    return rel_rms, mx


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def check_rows(gpu: np.ndarray, ref: np.ndarray, io: str, what=""):
    ref = np.asarray(ref, np.float64)
    gpu = np.asarray(gpu, np.float64)
    if io == "bf16":
        # the fp32 entry within 1e-4 * rms(row) of the oracle, then one rounding to bf16
        rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
        lim = 1e-4 * rms + 0.5 * bf16_ulp(ref) * 1.0001
        ok = np.abs(gpu - ref) <= lim
        assert ok.all(), f"{what}: {(~ok).sum()} bf16 values off"
    else:
        nrm = np.linalg.norm(ref, axis=-1)
        rel = np.linalg.norm(gpu - ref, axis=-1) / np.maximum(nrm, 1e-300)
        assert rel.max() <= 1e-4, f"{what}: row rel err {rel.max():.3e}"
        rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
        assert (np.abs(gpu - ref) <= 1e-4 * rms).all(), f"{what}: element err"
