"""Whole-workload driver of the float64 oracle (TEST INFRASTRUCTURE; see csa_oracle).

Takes a workload's input arrays (the bytes the CUDA path also reads) and its shape
constants (any object with the attributes of a workload shape: m, c, rope_dims,
rope_base, rms_eps, n_heads, n_idx_heads, d_idx, topk, n_win, n_cap, ctx, kind, io,
idx, B, T), decodes them with the oracle's own decoders and runs the steps of
csa_oracle for the requested queries, one query at a time.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional, Tuple

import numpy as np

from . import csa_oracle as O


def decode_indexer(s, inp) -> Tuple[np.ndarray, np.ndarray]:
    """Decoded indexer queries [B,T,H_I,d_I] and keys [B,N,d_I] in float64."""
    if s.idx == "f32":
        return np.asarray(inp["qI"], np.float64), np.asarray(inp["KI"], np.float64)
    if s.idx == "bf16":
        return O.dec_bf16(inp["qI"]), O.dec_bf16(inp["KI"])
    if s.idx == "fp8":
        return O.dec_bf16(inp["qI"]), O.dec_fp8_rows(inp["KI"], inp["KI_scale"])
    if s.idx == "mxfp4":
        return (O.dec_mxfp4(inp["qI"], inp["qI_scale"]),
                O.dec_mxfp4(inp["KI"], inp["KI_scale"]))
    raise ValueError(s.idx)


def compressed_cache(s, inp) -> np.ndarray:
    """The request-0 compressed KV cache [N, c] after this chunk's compression: rows before
    the chunk are the given prefix entries; the chunk's n_tok/m entries are compressed
    (overlapped, b-branch of the first block from the prefix tail when the chunk does
    not start the sequence) and finalised (RMSNorm + RoPE at m*i) [P1 1(1), 3(1), 3(2)].
    Decode workloads return the given cache."""
    kv = O.dec_io(inp["kv_cache"], s.io)
    if s.kind != "csa_prefill":
        return kv
    kv = kv.copy()
    first = s.ctx // s.m
    prev_Cb = O.dec_io(inp["prev_Cb"], s.io) if "prev_Cb" in inp else None
    prev_Zb = O.dec_io(inp["prev_Zb"], s.io) if "prev_Zb" in inp else None
    comp = O.compress_csa(O.dec_io(inp["Ca"], s.io), O.dec_io(inp["Cb"], s.io),
                          O.dec_io(inp["Za"], s.io), O.dec_io(inp["Zb"], s.io),
                          O.dec_io(inp["bias"], s.io), s.m, prev_Cb, prev_Zb)
    fin = O.finalize_entries(comp, first, s.m, s.rope_dims, s.rope_base, s.rms_eps)
    kv[0, first:first + fin.shape[0]] = fin
    return kv


def run(s, inp, queries: Optional[Iterable[Tuple[int, int]]] = None, *,
        idx_override: Optional[Dict[Tuple[int, int], np.ndarray]] = None,
        kv: Optional[np.ndarray] = None, want_scores: bool = True) -> Dict[str, dict]:
    """Run the oracle for the listed (b, t-index) queries (default: all).

    Returns {"scores": {(b,ti): [n_vis]}, "idx": {(b,ti): [k]}, "out": {(b,ti): [H,c]},
    "kv": the decoded (and, for prefill, freshly compressed) cache}. With ``idx_override``
    the attention of those queries uses the given selection instead of the oracle's own
    (used to compare the output of a CUDA selection that differs only at near-ties).
    """
    B, T = s.B, s.T
    if queries is None:
        queries = [(b, ti) for b in range(B) for ti in range(T)]
    queries = list(queries)
    kv = compressed_cache(s, inp) if kv is None else kv
    q = inp["q"]
    pos = np.asarray(inp["q_pos"], np.int64)
    win = inp["win_kv"]
    pos0 = np.asarray(inp["win_pos0"], np.int64)
    sink = np.asarray(inp["sink"], np.float64)
    scale = 1.0 / np.sqrt(s.c)
    res = {"scores": {}, "idx": {}, "out": {}, "kv": kv}
    qI = KI = None
    if s.kind in ("csa_prefill", "csa_decode"):
        qI, KI = decode_indexer(s, inp)
    for (b, ti) in queries:
        t = int(pos[b, ti])
        q_t = O.dec_io(q[b, ti], s.io)
        win_b = O.dec_io(win[b], s.io)
        n_vis = O.visible_entries(t, s.m, s.n_cap)
        if s.kind == "hca_decode":
            o = O.hca_query(q_t, t, kv[b], n_vis, win_b, int(pos0[b]), sink, r=s.rope_dims,
                            base=s.rope_base, eps=s.rms_eps, scale=scale, n_win=s.n_win)
        else:
            sc = O.index_scores(qI[b, ti], np.asarray(inp["w"][b, ti], np.float64), KI[b],
                                n_vis)
            sel = O.topk_select(sc, s.topk)
            if want_scores:
                res["scores"][(b, ti)] = sc
            res["idx"][(b, ti)] = sel
            use = sel if idx_override is None or (b, ti) not in idx_override \
                else idx_override[(b, ti)]
            o = O.csa_query(q_t, t, kv[b], use, win_b, int(pos0[b]), sink, r=s.rope_dims,
                            base=s.rope_base, eps=s.rms_eps, scale=scale, n_win=s.n_win)
        res["out"][(b, ti)] = o
    return res
