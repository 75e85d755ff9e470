"""The oracle's pins catch plausible mistakes.

Each case plants one slip in the float64 oracle (on the CPU, via monkeypatch) and
checks that at least one pin of test_oracle_pins fails against the mutated oracle.
"""
import inspect
import os

import numpy as np
import pytest

from oracle import csa_oracle as O
import tests.test_oracle_pins as PINS

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _pins():
    out = []
    for name, fn in sorted(vars(PINS).items()):
        if name.startswith("test_") and callable(fn):
            out.append(fn)
    return out


def _run_all_pins():
    """Run every pin; return the names of those that fail."""
    failed = []
    for fn in _pins():
        params = inspect.signature(fn).parameters
        calls = []
        if "branch" in params:
            calls = [dict(branch="a"), dict(branch="b")]
        elif "golden_dir" in params:
            calls = [dict(golden_dir=GOLDEN)]
        else:
            calls = [dict()]
        for kw in calls:
            try:
                fn(**kw)
            except (AssertionError, ValueError, IndexError):
                failed.append(fn.__name__)
                break
    return failed


def _mut_b_branch_same_block(Za, Zb, Ba, Bb, m, i, prev_Zb=None):
    za = Za[m * i:m * (i + 1)] + Ba
    zb = Zb[m * i:m * (i + 1)] + Bb  # wrong block for the b-branch
    return O._softmax_rows(np.concatenate([za, zb], axis=0))


def _mut_softmax_over_channels(logits):
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return e / e.sum(axis=1, keepdims=True)


def _mut_rope_freq(x, pos, r, base):
    x = np.array(x, np.float64, copy=True)
    if r == 0:
        return x
    c = x.shape[-1]
    p = np.arange(r // 2, dtype=np.float64)
    ang = np.asarray(pos, np.float64)[..., None] * base ** (-p / r)  # wrong exponent
    cos, sin = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., c - r::2].copy(), x[..., c - r + 1::2].copy()
    x[..., c - r::2] = x0 * cos - x1 * sin
    x[..., c - r + 1::2] = x0 * sin + x1 * cos
    return x


def _mut_rope_first_dims(x, pos, r, base):
    x = np.array(x, np.float64, copy=True)
    if r == 0:
        return x
    p = np.arange(r // 2, dtype=np.float64)
    ang = np.asarray(pos, np.float64)[..., None] * base ** (-2 * p / r)
    cos, sin = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0:r:2].copy(), x[..., 1:r:2].copy()  # rotates the first r dims
    x[..., 0:r:2] = x0 * cos - x1 * sin
    x[..., 1:r:2] = x0 * sin + x1 * cos
    return x


def _mut_unrotate_plus(o, t, r, base):
    return O.rope(o, +t, r, base)


def _mut_relu_after_weight(qI_t, w_t, KI, n_vis):
    dots = np.asarray(KI, np.float64)[:n_vis] @ np.asarray(qI_t, np.float64).T
    return np.maximum(dots * np.asarray(w_t, np.float64), 0.0).sum(axis=1)


def _mut_visibility_inclusive(t, m, n_cap):
    return max(0, min(t // m + 1, n_cap))


def _mut_sink_in_numerator(qh, rows, sink, scale):
    qh, rows = np.asarray(qh, np.float64), np.asarray(rows, np.float64)
    zs = np.full((qh.shape[0],), -np.inf) if sink is None else np.asarray(sink, np.float64)
    z = (qh @ rows.T) * scale
    M = np.maximum(z.max(axis=1), zs)
    e = np.exp(z - M[:, None])
    return (e @ rows) / e.sum(axis=1)[:, None]  # sink dropped from the denominator


def _mut_topk_ties_desc(scores, k):
    scores = np.asarray(scores, np.float64)
    n = scores.size
    order = sorted(range(n), key=lambda i: (-scores[i], -i))[:k]
    out = np.full((k,), -1, dtype=np.int64)
    out[:len(order)] = order
    return out


def _mut_rms_no_mean(x, eps, gamma=None):
    x = np.asarray(x, np.float64)
    y = x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
    return y if gamma is None else y * gamma


def _mut_window_excludes_query(t, n_win, pos0, l_raw):
    lo = max(t - n_win, 0)
    return np.arange(lo, t, dtype=np.int64)


MUTATIONS = {
    "b_branch_same_block": ("csa_pool_weights", _mut_b_branch_same_block),
    "softmax_over_channels": ("_softmax_rows", _mut_softmax_over_channels),
    "rope_frequency": ("rope", _mut_rope_freq),
    "rope_first_dims": ("rope", _mut_rope_first_dims),
    "unrotate_plus_t": ("output_unrotate", _mut_unrotate_plus),
    "relu_after_weight": ("index_scores", _mut_relu_after_weight),
    "visibility_inclusive": ("visible_entries", _mut_visibility_inclusive),
    "sink_dropped": ("core_attention", _mut_sink_in_numerator),
    "topk_ties_desc": ("topk_select", _mut_topk_ties_desc),
    "rms_sum_not_mean": ("rms_norm", _mut_rms_no_mean),
    "window_excludes_query": ("window_positions", _mut_window_excludes_query),
}


def test_unmutated_oracle_passes_every_pin():
    assert _run_all_pins() == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = _run_all_pins()
    assert failed, f"no pin caught the planted mistake {name}"


def test_e4m3_decoder_mutation_is_caught(monkeypatch):
    orig = O.dec_e4m3
    monkeypatch.setattr(O, "dec_e4m3", lambda c: orig(c) * 0.5)
    assert "test_e4m3_decoder_matches_torch_all_codes" in _run_all_pins()
