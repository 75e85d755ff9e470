"""Float64 CPU oracle of the CSA / HCA attention hot path (DeepSeek-V4 hybrid attention).

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference leg may import or run this module. The product (the CUDA
library ``libcsa.so`` and its Python binding) never calls it, and it shares no code
with the CUDA path: it decodes the input bytes itself and computes every step in
float64 with plain numpy, one function per step, in the order and notation of the
source pages.

Sources (cited by page title and section):
  [P1] 【论文解读】DeepSeek-V4 (wkq9411.github.io), 一、模型架构 (三) 混合注意力架构：CSA + HCA
       1(1) 压缩 KV Entries -- overlapped compression equations (Softmax_row, C_i^Comp);
       1(2) Lightning Indexer 稀疏选择 -- index score I_{t,s}, visibility s < Floor(t/m),
            Top-k selector C_t^SprsComp;
       1(3) Shared Key-Value MQA -- CoreAttn with key = value = selected entries;
       2(1) HCA 压缩 KV Entries -- non-overlapped compression (S, C_i^Comp);
       2(2) HCA Shared Key-Value MQA -- dense MQA over all entries;
       3(1) Query 和 KV Entry 的归一化 -- RMSNorm of each query head and of the KV entry;
       3(2) 部分 RoPE -- RoPE on the last 64 dims of q and KV, output rotated at position -t;
       3(3) 滑动窗口注意力 -- n_win uncompressed entries of the most recent tokens;
       3(4) Attention Sink -- exp(z'_h) added to the softmax denominator (s_{h,i,j}).
       1(4) 分组输出投影 -- n_h head outputs in g groups, each projected to d_g, then the
            g*d_g concatenation projected to d; 2(2) applies the same to HCA;
       4 效率分析 item 1 -- KV entries stored with the RoPE dims in BF16, the rest in FP8;
     二、基础设施 (四) FP4 量化感知训练 -- index scores quantised from FP32 to BF16 before
       the top-k selector (2x selector speed, 99.7% recall of the KV entries);
     三、预训练 (二) 模型配置 -- g = 8 / 16, d_g = 1024, d = 4096 / 7168.
  [P4] DeepseekV4论文解析 (blog.chaseai.de), 2. Hybrid Attention：CSA + HCA -- entry counts
       at 1M tokens (262,144 candidates; 1024+128 / 512+128 read; 8,192 + 128 for HCA);
       三、实验 -- the same precision split (RoPE dims BF16, rest FP8; BF16 index scores).

Readings where the pages leave a step open (each is a constant of the convention,
not a value the pages fix):
  R1  RoPE position of compressed entry i is m*i (first token of its a-block).
  R2  RoPE pairs adjacent dims (x_{2p}, x_{2p+1}) inside the last r dims, angle
      pos * base^(-2p/r), base 10000.
  R3  RMSNorm: x / sqrt(mean(x^2) + eps) * gamma, gamma = 1 unless given, eps = 1e-6;
      applied before RoPE.
  R4  Logit scale 1/sqrt(c) over all c dims.
  R5  A query at position t sees entries s < min(floor(t/m), N) (strict, as printed).
  R6  The window is the n_win most recent tokens including t itself: t-n_win+1 .. t;
      window rows are given in final (normed, rotated) form; no de-duplication against
      compressed entries.
  R7  Top-k order is (score descending, index ascending); slots beyond the visible
      count hold -1.
  R8  Indexer keys and queries get no RMSNorm / RoPE; the index score has no scale.
  R18 BF16 index scores: each score is rounded to the nearest bf16 value (ties to even)
      and the selector orders the rounded values by (value descending, index ascending).
  R19 Mixed-precision KV entry: the first c-r dims are FP8 e4m3 with one fp32 scale per
      entry row (amax/448, as for the FP8 indexer keys), the last r (RoPE) dims are bf16.
      Only compressed entries use it; sliding-window rows stay bf16.
  R20 Grouped output projection: group i holds heads i*H/g .. (i+1)*H/g-1, concatenated
      head after head; row vectors multiply weights from the left (x . W), as in the
      pages' projections; the input is the un-rotated attention output.
Parity of R1/R2 against the pages is unpinned (the pages fix neither); every other
step is pinned by the CPU tests (closed forms, invariants, brute force).
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

# ----------------------------------------------------------------------------
# decoders of the stored formats (written from the format definitions)
# ----------------------------------------------------------------------------


def dec_bf16(bits) -> np.ndarray:
    """bf16 bit patterns -> float64: the 16 bits are the top half of an IEEE binary32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def dec_io(x, io: str) -> np.ndarray:
    """Decode an activation tensor stored as fp32 or as bf16 bit patterns."""
    return dec_bf16(x) if io == "bf16" else np.asarray(x, np.float64)


def dec_e4m3(codes) -> np.ndarray:
    """OCP FP8 E4M3 ("fn"): sign, 4-bit exponent with bias 7, 3-bit fraction.

    Exponent field 0 is subnormal (f/8 * 2^-6); S.1111.111 is NaN; there is no infinity.
    """
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    f = (b & 7).astype(np.float64)
    mag = np.where(e == 0, (f / 8.0) * 2.0 ** -6, (1.0 + f / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (f == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def dec_e2m1(nib) -> np.ndarray:
    """OCP FP4 E2M1: sign, 2-bit exponent with bias 1, 1-bit fraction; exponent 0 is
    subnormal (f * 0.5). Magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}."""
    n = np.asarray(nib, dtype=np.int64)
    s = (n >> 3) & 1
    e = (n >> 1) & 3
    f = (n & 1).astype(np.float64)
    mag = np.where(e == 0, f * 0.5, (1.0 + f / 2.0) * np.exp2(e - 1.0))
    return np.where(s == 1, -mag, mag)


def dec_e8m0(b) -> np.ndarray:
    """OCP E8M0 scale: 2^(b - 127); 255 is NaN."""
    b = np.asarray(b, dtype=np.int64)
    return np.where(b == 255, np.nan, np.exp2(b - 127.0))


def dec_mxfp4(packed, scales) -> np.ndarray:
    """MXFP4 rows: packed e2m1 pairs (element 2j in the low nibble) with one e8m0 scale
    per 32 consecutive elements. Returns float64 [..., 2*packed.shape[-1]]."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = dec_e2m1(p & 0xF)
    hi = dec_e2m1(p >> 4)
    vals = np.stack([lo, hi], axis=-1).reshape(*p.shape[:-1], 2 * p.shape[-1])
    sc = dec_e8m0(scales)
    return vals * np.repeat(sc, 32, axis=-1)


def unblock_key_scales(blocked) -> np.ndarray:
    """MXFP4 key-cache scales are stored per block of 128 keys with byte 16*i + 4*j + b
    holding block-scale b of key 32*j + i. Returns them in key order [..., N, 4]."""
    sc = np.asarray(blocked, np.uint8)
    *lead, n, nb = sc.shape
    out = np.empty_like(sc)
    for blk in range(n // 128):
        for i in range(32):
            for j in range(4):
                out[..., 128 * blk + 32 * j + i, :] = sc[..., 128 * blk + 4 * i + j, :]
    return out


def dec_fp8_rows(codes, row_scale) -> np.ndarray:
    """FP8 e4m3 rows times their per-row fp32 scale."""
    return dec_e4m3(codes) * np.asarray(row_scale, np.float64)[..., None]


def dec_mixed_kv(nope_codes, nope_scale, rope_bits) -> np.ndarray:
    """Mixed-precision KV entry rows (reading R19) [P1 一(三)4 item 1]: FP8 e4m3 codes of
    the first c-r dims times the row's fp32 scale, followed by the last r (RoPE) dims as
    bf16. Returns float64 [..., c]."""
    return np.concatenate([dec_fp8_rows(nope_codes, nope_scale), dec_bf16(rope_bits)], axis=-1)


# ----------------------------------------------------------------------------
# stage 1: token-level KV compression  [P1 1(1), 2(1)]
# ----------------------------------------------------------------------------


def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    """Softmax over axis 0 (positions), separately for every channel (axis 1)."""
    mx = logits.max(axis=0, keepdims=True)
    e = np.exp(logits - mx)
    return e / e.sum(axis=0, keepdims=True)


def csa_pool_weights(Za, Zb, Ba, Bb, m: int, i: int, prev_Zb=None) -> np.ndarray:
    """[S^a_{mi..m(i+1)-1}; S^b_{m(i-1)..mi-1}] of entry i: a [2m, c] softmax over the 2m
    logits of each channel [P1 1(1), Softmax_row]. Block 0 without a preceding state pads
    the b-logits with -inf."""
    za = Za[m * i:m * (i + 1)] + Ba
    if i > 0:
        zb = Zb[m * (i - 1):m * i] + Bb
    elif prev_Zb is not None:
        zb = prev_Zb + Bb
    else:
        zb = np.full_like(za, -np.inf)
    return _softmax_rows(np.concatenate([za, zb], axis=0))


def compress_csa(Ca, Cb, Za, Zb, bias, m: int, prev_Cb=None, prev_Zb=None) -> np.ndarray:
    """Overlapped compression [P1 1(1)]: entry i = sum_j S^a_j * C^a_j over block i plus
    sum_j S^b_j * C^b_j over block i-1, the 2m weights softmax-normalised per channel.

    ``bias`` is [2m, c]: rows 0..m-1 are B^a, rows m..2m-1 are B^b (row r = offset r in
    the block). For i = 0 the b-branch comes from ``prev_*`` (the last m tokens before
    this chunk) when given, else its logits are -inf and its values 0 (sequence start).
    """
    Ca, Cb, Za, Zb, bias = (np.asarray(x, np.float64) for x in (Ca, Cb, Za, Zb, bias))
    n, c = Ca.shape
    assert n % m == 0
    Ba, Bb = bias[:m], bias[m:2 * m]
    out = np.empty((n // m, c))
    for i in range(n // m):
        S = csa_pool_weights(Za, Zb, Ba, Bb, m, i, prev_Zb)
        ca = Ca[m * i:m * (i + 1)]
        if i > 0:
            cb = Cb[m * (i - 1):m * i]
        elif prev_Cb is not None:
            cb = np.asarray(prev_Cb, np.float64)
        else:
            cb = np.zeros_like(ca)
        out[i] = (S[:m] * ca).sum(axis=0) + (S[m:] * cb).sum(axis=0)
    return out


def compress_hca(C, Z, bias, m: int) -> np.ndarray:
    """Non-overlapped compression [P1 2(1)]: entry i = sum_j S_j * C_j over the m' tokens of
    block i, S the per-channel softmax of Z_{m'i..m'(i+1)-1} + B."""
    C, Z, bias = (np.asarray(x, np.float64) for x in (C, Z, bias))
    n, c = C.shape
    assert n % m == 0
    out = np.empty((n // m, c))
    for i in range(n // m):
        S = _softmax_rows(Z[m * i:m * (i + 1)] + bias)
        out[i] = (S * C[m * i:m * (i + 1)]).sum(axis=0)
    return out


# ----------------------------------------------------------------------------
# normalisation and partial RoPE  [P1 3(1), 3(2)]
# ----------------------------------------------------------------------------


def rms_norm(x, eps: float, gamma=None) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma (reading R3)."""
    x = np.asarray(x, np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if gamma is None else y * np.asarray(gamma, np.float64)


def rope(x, pos, r: int, base: float) -> np.ndarray:
    """Rotate the last r dims of x (pairs (2p, 2p+1) of that slice) by pos * base^(-2p/r)
    (reading R2). ``pos`` is a scalar or broadcasts against x's leading axes."""
    x = np.array(x, np.float64, copy=True)
    if r == 0:
        return x
    c = x.shape[-1]
    p = np.arange(r // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * p / r)
    ang = np.asarray(pos, np.float64)[..., None] * inv_freq  # [..., r/2]
    cos, sin = np.cos(ang), np.sin(ang)
    x0 = x[..., c - r + 0::2].copy()
    x1 = x[..., c - r + 1::2].copy()
    x[..., c - r + 0::2] = x0 * cos - x1 * sin
    x[..., c - r + 1::2] = x0 * sin + x1 * cos
    return x


def finalize_entries(C, first_entry: int, m: int, r: int, base: float, eps: float,
                     gamma=None) -> np.ndarray:
    """KV entry head: RMSNorm, then RoPE at the entry's position m*(first_entry+i)
    (readings R1, R3) [P1 3(1), 3(2)]."""
    C = np.asarray(C, np.float64)
    pos = m * (first_entry + np.arange(C.shape[0], dtype=np.float64))
    return rope(rms_norm(C, eps, gamma), pos, r, base)


# ----------------------------------------------------------------------------
# stage 2 + 3: lightning indexer and top-k  [P1 1(2)]
# ----------------------------------------------------------------------------


def visible_entries(t: int, m: int, n_cap: int) -> int:
    """Number of compressed entries query t may see: s < floor(t/m), capped by the cache
    length (reading R5) [P1 1(2)]."""
    return max(0, min(t // m, n_cap))


def index_scores(qI_t, w_t, KI, n_vis: int) -> np.ndarray:
    """I_{t,s} = sum_h w_{t,h} * ReLU(q^I_{t,h} . K^IComp_s) for s < n_vis [P1 1(2)].

    qI_t [H_I, d_I], w_t [H_I], KI [N, d_I] (already decoded)."""
    qI_t = np.asarray(qI_t, np.float64)
    K = np.asarray(KI, np.float64)[:n_vis]
    dots = K @ qI_t.T  # [n_vis, H_I]: q_{t,h} . K_s
    return np.maximum(dots, 0.0) @ np.asarray(w_t, np.float64)


def index_score_scale(qI_t, w_t, KI, n_vis: int) -> np.ndarray:
    """sum_h |w_{t,h}| * ReLU(q^I_{t,h} . K_s): the sum of the magnitudes of the terms that
    make up I_{t,s}. Not part of the method: it is the scale against which a floating-point
    evaluation of I is compared (a rounding error of a sum grows with this, not with |I|,
    when signed head weights cancel). Equals |I| when every w >= 0."""
    qI_t = np.asarray(qI_t, np.float64)
    K = np.asarray(KI, np.float64)[:n_vis]
    return np.maximum(K @ qI_t.T, 0.0) @ np.abs(np.asarray(w_t, np.float64))


def topk_select(scores, k: int) -> np.ndarray:
    """Top-k of I_{t,:}: indices ordered by (score desc, index asc); slots past the
    number of candidates hold -1 (reading R7) [P1 1(2), C_t^SprsComp]."""
    scores = np.asarray(scores, np.float64)
    order = np.argsort(-scores, kind="stable")[:k]
    out = np.full((k,), -1, dtype=np.int64)
    out[:order.size] = order
    return out


def round_to_bf16(x) -> np.ndarray:
    """Nearest bf16 value of each x (8 significant bits, ties to the even significand),
    computed from the format's definition: with e = floor(log2|x|) (at least -126, bf16's
    smallest normal exponent) the bf16 values near x are the multiples of 2^(e-7).
    Finite inputs whose rounded value stays finite; zero stays zero."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    ulp = np.exp2(e - 7.0)
    return np.rint(x / ulp) * ulp  # np.rint rounds halves to even


def topk_select_bf16(scores, k: int) -> np.ndarray:
    """Top-k on BF16 index scores (reading R18) [P1 二(四)]: the selector of
    ``topk_select`` applied to the scores rounded to bf16, so that scores rounding to the
    same bf16 value tie and the smaller index wins."""
    return topk_select(round_to_bf16(scores), k)


# ----------------------------------------------------------------------------
# stage 4: shared-KV MQA with window and sink  [P1 1(3), 3(1)-(4)]
# ----------------------------------------------------------------------------


def query_prep(q_t, t: int, r: int, base: float, eps: float, gamma=None) -> np.ndarray:
    """Per query head: RMSNorm, then RoPE at position t [P1 3(1), 3(2)]. q_t [H, c]."""
    return rope(rms_norm(q_t, eps, gamma), t, r, base)


def window_positions(t: int, n_win: int, pos0: int, l_raw: int) -> np.ndarray:
    """Token positions of query t's window: max(t-n_win+1, 0) .. t (reading R6). The
    caller's window buffer must hold them (rows pos0 .. pos0+l_raw-1)."""
    lo = max(t - n_win + 1, 0)
    if n_win <= 0:
        return np.zeros((0,), np.int64)
    assert lo >= pos0 and t < pos0 + l_raw, "window buffer does not cover the query"
    return np.arange(lo, t + 1, dtype=np.int64)


def core_attention(qh, rows, sink, scale: float) -> np.ndarray:
    """o_h = sum_j exp(z_j) v_j / (sum_j exp(z_j) + exp(z'_h)) with z_j = scale * q_h . k_j
    and v_j = k_j (key = value) [P1 1(3) CoreAttn; 3(4) sink equation s_{h,i,j}].

    qh [H, c], rows [L, c], sink [H] or None (no sink = z' = -inf). Computed with the max
    of all logits (sink included) subtracted, which leaves the ratio unchanged."""
    qh = np.asarray(qh, np.float64)
    rows = np.asarray(rows, np.float64)
    H = qh.shape[0]
    zs = np.full((H,), -np.inf) if sink is None else np.asarray(sink, np.float64)
    if rows.shape[0] == 0:
        return np.zeros_like(qh)
    z = (qh @ rows.T) * scale  # [H, L]
    M = np.maximum(z.max(axis=1), zs)
    e = np.exp(z - M[:, None])
    den = e.sum(axis=1) + np.exp(zs - M)
    return (e @ rows) / den[:, None]


def output_unrotate(o, t: int, r: int, base: float) -> np.ndarray:
    """RoPE at position -t on the last r dims of every head's output [P1 3(2)]."""
    return rope(o, -t, r, base)


def csa_query(q_t, t: int, kv_rows, idx, win_kv, pos0: int, sink, *, r: int, base: float,
              eps: float, scale: float, n_win: int, q_gamma=None) -> np.ndarray:
    """Output [H, c] of one CSA query: prep q, attend over the selected entries followed by
    the window rows, un-rotate [P1 1(3), 3(1)-(4)]. ``kv_rows`` is the request's decoded
    compressed cache, ``idx`` its top-k list (-1 entries skipped)."""
    qh = query_prep(q_t, t, r, base, eps, q_gamma)
    sel = np.asarray([int(i) for i in idx if i >= 0], dtype=np.int64)
    win = np.asarray(win_kv, np.float64)
    wp = window_positions(t, n_win, pos0, win.shape[0])
    rows = np.concatenate([np.asarray(kv_rows, np.float64)[sel], win[wp - pos0]], axis=0)
    return output_unrotate(core_attention(qh, rows, sink, scale), t, r, base)


def hca_query(q_t, t: int, kv_rows, n_vis: int, win_kv, pos0: int, sink, *, r: int,
              base: float, eps: float, scale: float, n_win: int, q_gamma=None) -> np.ndarray:
    """Output [H, c] of one HCA query: dense MQA over all n_vis visible entries plus the
    window [P1 2(2), 3(1)-(4)]."""
    qh = query_prep(q_t, t, r, base, eps, q_gamma)
    win = np.asarray(win_kv, np.float64)
    wp = window_positions(t, n_win, pos0, win.shape[0])
    rows = np.concatenate([np.asarray(kv_rows, np.float64)[:n_vis], win[wp - pos0]], axis=0)
    return output_unrotate(core_attention(qh, rows, sink, scale), t, r, base)


def default_scale(c: int) -> float:
    """Logit scale 1/sqrt(c) (reading R4)."""
    return 1.0 / math.sqrt(c)


# ----------------------------------------------------------------------------
# grouped output projection  [P1 1(4), 2(2)]
# ----------------------------------------------------------------------------


def grouped_output_projection(o_t, w_grp, w_out) -> np.ndarray:
    """Attention output of one query [P1 1(4) 分组输出投影] (reading R20).

    o_t [H, c]: the un-rotated core-attention outputs o_{t,1..H}.
    w_grp [g, c*H/g, d_g]: group i's projection of o^G_{t,i} (heads i*H/g .. (i+1)*H/g-1,
    concatenated) to the intermediate output o^G'_{t,i}.
    w_out [g*d_g, d]: projection of [o^G'_{t,1}; ...; o^G'_{t,g}] to the output.
    Returns [d]."""
    o_t = np.asarray(o_t, np.float64)
    w_grp = np.asarray(w_grp, np.float64)
    w_out = np.asarray(w_out, np.float64)
    H, c = o_t.shape
    g, width, d_g = w_grp.shape
    assert H % g == 0 and width == c * (H // g) and w_out.shape[0] == g * d_g
    hg = H // g
    mid = np.empty((g, d_g))
    for i in range(g):
        o_group = o_t[i * hg:(i + 1) * hg].reshape(width)  # o^G_{t,i}
        mid[i] = o_group @ w_grp[i]                          # o^G'_{t,i}
    return mid.reshape(g * d_g) @ w_out

