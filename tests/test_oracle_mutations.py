"""The oracle's pins catch plausible mistakes.

Each case plants one slip in the float64 oracle (on the CPU, via monkeypatch) and
checks that at least one pin of test_oracle_pins or test_oracle_next_pins fails against
the mutated oracle.
"""
import inspect
import os

import numpy as np
import pytest

from oracle import csa_oracle as O
from oracle import state_cache as SC
import tests.test_oracle_next_pins as NEXT_PINS
import tests.test_oracle_pins as PINS

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _pins():
    out = []
    for mod in (PINS, NEXT_PINS):
        for name, fn in sorted(vars(mod).items()):
            if name.startswith("test_") and callable(fn):
                out.append(fn)
    return out


def _calls(fn):
    """Keyword sets to call a pin with: its parametrize marks expanded, the golden folder
    supplied."""
    calls = [dict()]
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names = [n.strip() for n in mark.args[0].split(",")] if isinstance(mark.args[0], str) \
            else list(mark.args[0])
        rows = [v if len(names) > 1 else (v,) for v in mark.args[1]]
        calls = [dict(c, **dict(zip(names, row))) for c in calls for row in rows]
    if "golden_dir" in inspect.signature(fn).parameters:
        calls = [dict(c, golden_dir=GOLDEN) for c in calls]
    return calls


def _run_all_pins():
    """Run every pin; return the names of those that fail."""
    failed = []
    for fn in _pins():
        for kw in _calls(fn):
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
    with np.errstate(invalid="ignore"):  # rows of -inf (a sequence start) give NaN here
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


def _bf16_ulp(x):
    a = np.abs(np.asarray(x, np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.exp2(np.maximum(e, -126.0) - 7.0)


def _mut_bf16_truncate(x):
    u = _bf16_ulp(x)
    return np.trunc(np.asarray(x, np.float64) / u) * u


def _mut_bf16_ties_away(x):
    x = np.asarray(x, np.float64)
    u = _bf16_ulp(x)
    return np.sign(x) * np.floor(np.abs(x) / u + 0.5) * u


def _mut_mixed_kv_rope_first(nope_codes, nope_scale, rope_bits):
    return np.concatenate([O.dec_bf16(rope_bits), O.dec_fp8_rows(nope_codes, nope_scale)], -1)


def _mut_mixed_kv_no_scale(nope_codes, nope_scale, rope_bits):
    return np.concatenate([O.dec_e4m3(nope_codes), O.dec_bf16(rope_bits)], -1)


def _mut_groups_interleaved(o_t, w_grp, w_out):
    o_t = np.asarray(o_t, np.float64)
    g = w_grp.shape[0]
    mid = np.stack([o_t[i::g].reshape(-1) @ w_grp[i] for i in range(g)])  # heads i, i+g, ..
    return mid.reshape(-1) @ w_out


def _mut_groups_concat_transposed(o_t, w_grp, w_out):
    o_t = np.asarray(o_t, np.float64)
    g = w_grp.shape[0]
    hg = o_t.shape[0] // g
    mid = np.stack([o_t[i * hg:(i + 1) * hg].reshape(-1) @ w_grp[i] for i in range(g)])
    return mid.T.reshape(-1) @ w_out  # [d_g, g] order instead of [g, d_g]


def _mut_state_forgets_b_rows(self):
    return np.full((self.m, self.c), -np.inf), np.zeros((self.m, self.c))


def _mut_state_position_off_by_one(self, entry, i):
    return O.finalize_entries(entry[None], i + 1, self.m, self.r, self.base, self.eps,
                              self.gamma)[0]


def _mut_ring_slot_shifted(self, row, pos):
    if self.n_win > 0:
        self.ring[(pos + 1) % self.n_win] = np.asarray(row, np.float64)


def _mut_release_leaks(self):
    self.page_table = []


def _mut_resume_wrong_block(self, Ca, Cb, Za, Zb, entries, win_rows):
    # takes the open block's b-rows as the last finished block's
    assert self.n_tok == 0 and self.n_entries == 0
    Ca, Cb, Za, Zb = (np.asarray(x, np.float64) for x in (Ca, Cb, Za, Zb))
    n0 = Ca.shape[0]
    nb = n0 // self.m
    for row in entries:
        self._write_entry(np.asarray(row, np.float64))
    if nb > 0:
        lo = min(self.m * nb, n0 - self.m)
        self.prev_Cb, self.prev_Zb = Cb[lo:lo + self.m].copy(), Zb[lo:lo + self.m].copy()
    tail = slice(self.m * nb, n0)
    self.cur = {"Ca": list(Ca[tail]), "Za": list(Za[tail]), "Cb": list(Cb[tail]),
                "Zb": list(Zb[tail])}
    win_rows = np.asarray(win_rows, np.float64)
    for p in range(max(n0 - self.n_win, 0), n0):
        self._push_window(win_rows[p], p)
    self.n_tok = n0


def _mut_hca_bias_on_values(self, cv, zv, win_row):
    t = self.n_tok
    self.cur_C.append(np.asarray(cv, np.float64))
    self.cur_Z.append(np.asarray(zv, np.float64))
    self._push_window(win_row, t)
    self.n_tok += 1
    if self.n_tok % self.m:
        return None
    i = t // self.m
    S = O._softmax_rows(np.stack(self.cur_Z))
    entry = (S * (np.stack(self.cur_C) + self.B)).sum(axis=0)  # bias on the values
    if self.finalize:
        entry = O.finalize_entries(entry[None], i, self.m, self.r, self.base, self.eps,
                                   self.gamma)[0]
    self._write_entry(entry)
    self.cur_C, self.cur_Z = [], []
    return i


NEXT_MUTATIONS = {
    "resume_takes_open_block_b_rows": (SC.CsaState, "resume", _mut_resume_wrong_block),
    "hca_bias_on_values": (SC.HcaState, "append", _mut_hca_bias_on_values),
    "bf16_truncates": (O, "round_to_bf16", _mut_bf16_truncate),
    "bf16_ties_away_from_zero": (O, "round_to_bf16", _mut_bf16_ties_away),
    "bf16_scores_not_rounded": (O, "topk_select_bf16", lambda s, k: O.topk_select(s, k)),
    "mixed_kv_rope_dims_first": (O, "dec_mixed_kv", _mut_mixed_kv_rope_first),
    "mixed_kv_scale_dropped": (O, "dec_mixed_kv", _mut_mixed_kv_no_scale),
    "output_groups_interleaved": (O, "grouped_output_projection", _mut_groups_interleaved),
    "output_groups_concat_transposed": (O, "grouped_output_projection",
                                        _mut_groups_concat_transposed),
    "state_forgets_b_rows": (SC.CsaState, "_b_branch", _mut_state_forgets_b_rows),
    "state_entry_position_off_by_one": (SC.CsaState, "_finalize", _mut_state_position_off_by_one),
    "window_ring_slot_shifted": (SC._Request, "_push_window", _mut_ring_slot_shifted),
    "release_leaks_pages": (SC._Request, "release", _mut_release_leaks),
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


@pytest.mark.parametrize("name", sorted(NEXT_MUTATIONS))
def test_next_step_mutation_is_caught(name, monkeypatch):
    owner, attr, fn = NEXT_MUTATIONS[name]
    monkeypatch.setattr(owner, attr, fn)
    failed = _run_all_pins()
    assert failed, f"no pin caught the planted mistake {name}"
