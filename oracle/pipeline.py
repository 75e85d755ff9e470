"""Whole-workload driver of the float64 oracle (TEST INFRASTRUCTURE; see csa_oracle).

Takes a workload's input arrays (the bytes the CUDA path also reads) and its shape
constants (any object with the attributes of a workload shape: m, c, rope_dims,
rope_base, rms_eps, n_heads, n_idx_heads, d_idx, topk, n_win, n_cap, ctx, kind, io,
idx, B, T, n_tok), decodes them with the oracle's own decoders and runs the steps of
csa_oracle for the requested queries, one query at a time. Large caches are decoded
per request, and compressed-KV rows only where a query reads them.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional, Tuple

import numpy as np

from . import csa_oracle as O


def decode_indexer_request(s, inp, b: int) -> Tuple[np.ndarray, np.ndarray]:
    """Decoded indexer queries [T,H_I,d_I] and keys [N,d_I] of request b, float64."""
    if s.idx == "f32":
        return np.asarray(inp["qI"][b], np.float64), np.asarray(inp["KI"][b], np.float64)
    if s.idx == "bf16":
        return O.dec_bf16(inp["qI"][b]), O.dec_bf16(inp["KI"][b])
    if s.idx == "fp8":
        return O.dec_bf16(inp["qI"][b]), O.dec_fp8_rows(inp["KI"][b], inp["KI_scale"][b])
    if s.idx == "mxfp4":
        return (O.dec_mxfp4(inp["qI"][b], inp["qI_scale"][b]),
                O.dec_mxfp4(inp["KI"][b], O.unblock_key_scales(inp["KI_scale"][b])))
    raise ValueError(s.idx)


def compressed_chunk(s, inp) -> np.ndarray:
    """The chunk's new entries [B, n_tok/m, c] of a prefill workload: overlapped compression
    (the first block's b-branch from the prefix tail when the chunk does not start the
    sequence) then RMSNorm + RoPE at m*i [P1 1(1), 3(1), 3(2)]."""
    first = s.ctx // s.m
    prev_Cb = O.dec_io(inp["prev_Cb"], s.io) if "prev_Cb" in inp else None
    prev_Zb = O.dec_io(inp["prev_Zb"], s.io) if "prev_Zb" in inp else None
    comp = O.compress_csa(O.dec_io(inp["Ca"], s.io), O.dec_io(inp["Cb"], s.io),
                          O.dec_io(inp["Za"], s.io), O.dec_io(inp["Zb"], s.io),
                          O.dec_io(inp["bias"], s.io), s.m, prev_Cb, prev_Zb)
    fin = O.finalize_entries(comp, first, s.m, s.rope_dims, s.rope_base, s.rms_eps)
    return fin[None]


class _Cache:
    """Row access to request b's compressed cache, decoding only the rows asked for. A cache
    given as mixed-precision rows (inputs kv_codes, kv_scale, kv_rope instead of kv_cache)
    is decoded with dec_mixed_kv."""

    def __init__(self, s, inp, chunk: Optional[np.ndarray]):
        self.s, self.chunk = s, chunk
        self.mixed = "kv_scale" in inp
        if self.mixed:
            self.codes, self.kscale, self.rope = inp["kv_codes"], inp["kv_scale"], inp["kv_rope"]
        else:
            self.raw = inp["kv_cache"]
        self.first = s.ctx // s.m if chunk is not None else None

    def rows(self, b: int, sel: np.ndarray) -> np.ndarray:
        sel = np.asarray(sel, np.int64)
        if not sel.size:
            out = np.zeros((0, self.s.c))
        elif self.mixed:
            out = O.dec_mixed_kv(self.codes[b][sel], self.kscale[b][sel], self.rope[b][sel])
        else:
            out = O.dec_io(self.raw[b][sel], self.s.io)
        if self.chunk is not None and sel.size:
            n_new = self.chunk.shape[1]
            inside = (sel >= self.first) & (sel < self.first + n_new)
            out[inside] = self.chunk[b, sel[inside] - self.first]
        return out


def run(s, inp, queries: Optional[Iterable[Tuple[int, int]]] = None, *,
        idx_override: Optional[Dict[Tuple[int, int], np.ndarray]] = None,
        want_scores: bool = True) -> Dict[str, dict]:
    """Run the oracle for the listed (b, t-index) queries (default: all).

    Returns {"scores": {(b,ti): [n_vis]}, "scale": {(b,ti): [n_vis]} (the magnitude sums of
    index_score_scale), "idx": {(b,ti): [k]}, "out": {(b,ti): [H,c]}, "chunk": the freshly
    compressed entries of a prefill chunk (or None)}. With
    ``idx_override`` the attention of those queries uses the given selection instead of
    the oracle's own (to compare the output of a CUDA selection that differs from the
    oracle's only at near-ties).
    """
    B, T = s.B, s.T
    if queries is None:
        queries = [(b, ti) for b in range(B) for ti in range(T)]
    queries = sorted(queries)
    chunk = compressed_chunk(s, inp) if s.kind == "csa_prefill" else None
    cache = _Cache(s, inp, chunk)
    pos = np.asarray(inp["q_pos"], np.int64)
    pos0 = np.asarray(inp["win_pos0"], np.int64)
    sink = np.asarray(inp["sink"], np.float64)
    scale = 1.0 / np.sqrt(s.c)
    res = {"scores": {}, "scale": {}, "idx": {}, "out": {}, "chunk": chunk}
    cur_b, qI_b, KI_b = None, None, None
    for (b, ti) in queries:
        t = int(pos[b, ti])
        q_t = O.dec_io(inp["q"][b, ti], s.io)
        win_b = O.dec_io(inp["win_kv"][b], s.io)
        n_vis = O.visible_entries(t, s.m, s.n_cap)
        if s.kind == "hca_decode":
            rows = cache.rows(b, np.arange(n_vis))
            o = O.hca_query(q_t, t, rows, n_vis, win_b, int(pos0[b]), sink, r=s.rope_dims,
                            base=s.rope_base, eps=s.rms_eps, scale=scale, n_win=s.n_win)
        else:
            given = idx_override is not None and (b, ti) in idx_override
            if given and not want_scores:  # attention only, on the given selection
                use = np.asarray(idx_override[(b, ti)], np.int64)
            else:
                if b != cur_b:
                    qI_b, KI_b = decode_indexer_request(s, inp, b)
                    cur_b = b
                sc = O.index_scores(qI_b[ti], np.asarray(inp["w"][b, ti], np.float64), KI_b,
                                    n_vis)
                sel = O.topk_select(sc, s.topk)
                if want_scores:
                    res["scores"][(b, ti)] = sc
                    res["scale"][(b, ti)] = O.index_score_scale(
                        qI_b[ti], np.asarray(inp["w"][b, ti], np.float64), KI_b, n_vis)
                res["idx"][(b, ti)] = sel
                use = np.asarray(idx_override[(b, ti)], np.int64) if given else sel
            valid = use[(use >= 0) & (use < s.n_cap)]
            rows = cache.rows(b, valid)
            o = O.csa_query(q_t, t, rows, np.arange(valid.size), win_b, int(pos0[b]), sink,
                            r=s.rope_dims, base=s.rope_base, eps=s.rms_eps, scale=scale,
                            n_win=s.n_win)
        res["out"][(b, ti)] = o
    return res
