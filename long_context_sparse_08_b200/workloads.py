"""Seeded synthetic inputs for the CSA / HCA hot path, and their storage encodings.

This module draws random numbers and encodes them into the byte formats the
library consumes (bf16, FP8 e4m3 with a per-row fp32 scale, MXFP4 = e2m1
values with one e8m0 scale per 32 elements). It holds none of the attention
method's arithmetic: no compression, scoring, selection or attention. Both the
CUDA path and the float64 oracle read the bytes produced here, each with its own
decoder.

Workload shapes follow the model configuration table of 【论文解读】DeepSeek-V4
(三、预训练 (二) 模型配置: m=4, m'=128, n_h^I=64, c^I=128, top-k 512/1024,
n_h 64/128, c=512, n_win=128) and the 1M-token counts of DeepseekV4论文解析
(2. Hybrid Attention: 262,144 CSA candidates, 8,192 HCA entries).

Generator: numpy ``Generator(PCG64(seed))``. Tensors are drawn in the order
``make_inputs`` lists them for each workload kind (the tensors a workload names first,
then the extras it needs, then the sink logits); fp32 draws are then encoded.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

# ----------------------------------------------------------------------------
# storage encodings (round-to-nearest-even with saturation)
# ----------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even. Finite inputs only.

    Works in uint32 (finite patterns stay below 2^32 after the rounding add) and in
    slices of 2^24 elements to bound temporary memory."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1).view(np.uint32)
    out = np.empty(flat.shape, np.uint16)
    step = 1 << 24
    for i in range(0, flat.size, step):
        u = flat[i:i + step]
        out[i:i + step] = ((u + (np.uint32(0x7FFF) + ((u >> 16) & np.uint32(1)))) >> 16)
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# e4m3 (OCP FP8, "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa, max 448.
_E4M3_MAX = 448.0


def quant_fp8_rowwise(x: np.ndarray):
    """Row-wise FP8 e4m3: scale = amax(row)/448 (fp32); codes = RNE(x/scale), saturating.

    Returns (codes uint8 [..., d], scale float32 [...]). A zero row gets scale 0 and
    all-zero codes.
    """
    import torch

    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = (amax / np.float32(_E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    y = (x / safe[..., None]).astype(np.float32)
    y = np.clip(y, -_E4M3_MAX, _E4M3_MAX)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def quant_mixed_kv(x: np.ndarray, r: int):
    """Mixed-precision KV entry rows: the first d-r dims row-wise FP8 e4m3 (scale =
    amax/448 over those dims), the last r dims bf16 (RNE).

    Returns (codes uint8 [..., d-r], scale float32 [...], rope bf16 bits uint16 [..., r]).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[-1]
    assert 0 < r < d
    codes, scale = quant_fp8_rowwise(x[..., :d - r])
    return codes, scale, f32_to_bf16_bits(np.ascontiguousarray(x[..., d - r:]))


# e2m1 grid (magnitudes) and their 3-bit codes (exponent 2 bits bias 1, mantissa 1 bit)
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def _e2m1_round_codes(v: np.ndarray) -> np.ndarray:
    """|v| -> nearest e2m1 magnitude code (0..7), ties to the even code, saturating at 6."""
    a = np.minimum(np.abs(v), 6.0).astype(np.float32)
    # midpoints between consecutive grid values; at a tie pick the even code
    mids = (_E2M1_GRID[1:] + _E2M1_GRID[:-1]) * 0.5  # 0.25 .75 1.25 1.75 2.5 3.5 5
    code = np.searchsorted(mids, a, side="left").astype(np.int64)  # a<=mid -> lower code
    tie = np.zeros_like(a, dtype=bool)
    for i, mval in enumerate(mids):
        tie |= a == mval
    # at an exact midpoint searchsorted(side=left) gave the lower code i; move to the even one
    lower = code
    upper = np.minimum(code + 1, 7)
    code = np.where(tie & (lower % 2 == 1), upper, lower)
    return code.astype(np.uint8)


def quant_mxfp4(x: np.ndarray):
    """MXFP4 encoding (OCP Microscaling v1.0 rule) along the last axis.

    Per block of 32: shared exponent E = floor(log2(amax)) - 2 (2 = e2m1's largest
    exponent), clamped to e8m0's range; elements are x / 2^E rounded to the e2m1 grid
    (RNE, saturating at +-6). An all-zero block gets E = -127.

    Returns (packed uint8 [..., d/2]; element 2j in the low nibble, 2j+1 in the high
    nibble) and (scales uint8 [..., d/32], e8m0 biased by 127).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[-1]
    assert d % 32 == 0
    xb = x.reshape(*x.shape[:-1], d // 32, 32)
    amax = np.abs(xb).max(axis=-1)
    with np.errstate(divide="ignore"):
        e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, -127)
    e = np.clip(e, -127, 127).astype(np.int64)
    scale = np.ldexp(np.float32(1.0), e).astype(np.float32)
    v = xb / scale[..., None]
    mag = _e2m1_round_codes(v)
    sign = ((v < 0) & (mag > 0)).astype(np.uint8)
    codes = (sign << 3) | mag  # 4-bit codes
    codes = codes.reshape(*x.shape[:-1], d)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, (e + 127).astype(np.uint8)


def block_key_scales(scales: np.ndarray) -> np.ndarray:
    """Key-cache scale layout: per block of 128 keys, byte 16*i + 4*j + b holds block-scale b
    of key 32*j + i (the layout tcgen05.cp copies into TMEM). Input [..., N, 4] in key
    order (N a multiple of 128); output has the same shape, reordered within blocks."""
    sc = np.ascontiguousarray(scales, np.uint8)
    *lead, n, nb = sc.shape
    assert n % 128 == 0 and nb == 4
    blk = sc.reshape(*lead, n // 128, 4, 32, 4)          # [.., blk, j, i, b]
    return np.ascontiguousarray(np.swapaxes(blk, -3, -2)).reshape(*lead, n, 4)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Shape:
    """Problem shape and method constants of one workload (plain numbers)."""

    name: str
    kind: str  # "csa_prefill" | "csa_decode" | "hca_decode" | "csa_compress" | "hca_compress"
    io: str  # "f32" | "bf16": dtype of q, KV rows and outputs
    idx: str  # indexer key format: "f32" | "bf16" | "fp8" | "mxfp4" | "none"
    B: int
    T: int  # queries per request
    m: int
    c: int
    rope_dims: int
    n_heads: int
    n_idx_heads: int
    d_idx: int
    topk: int
    n_win: int
    n_cap: int  # compressed-entry capacity of the cache
    ctx: int  # decode: tokens before the query; prefill: tokens before the chunk
    n_tok: int = 0  # per-token compression inputs (prefill / compress cases)
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    seed: int = 0
    w_dist: str = "normal"  # indexer head weights: "normal" | "uniform01"
    sink: str = "normal"  # "normal" | "zero"
    bias_std: float = 1.0
    overlap: int = 1
    q_pos_override: tuple = ()  # explicit per-request decode positions (edge cases)
    # degenerate selections: requests whose indexer head weights are all zero (every score
    # 0: the whole row ties), and a request whose indexer keys repeat with this period
    # (groups of equal scores at distinct indices)
    w_zero_requests: tuple = ()
    dup_keys: tuple = ()  # (request, period)


SHAPES: Dict[str, Shape] = {}


def _reg(s: Shape) -> Shape:
    SHAPES[s.name] = s
    return s


# Tiny CSA prefill, fp32: 256 tokens, every token a causal query.
TINY = _reg(Shape("tiny_prefill_f32", "csa_prefill", "f32", "f32", B=1, T=256, m=4, c=64,
                  rope_dims=16, n_heads=4, n_idx_heads=4, d_idx=32, topk=16, n_win=32,
                  n_cap=64, ctx=0, n_tok=256, seed=0, w_dist="uniform01", sink="zero",
                  bias_std=0.1))
# Flash-shaped CSA decode: B=8, 131072-token context, FP8 row-scaled indexer keys.
FLASH_DECODE = _reg(Shape("flash_decode_131k", "csa_decode", "bf16", "fp8", B=8, T=1, m=4,
                          c=512, rope_dims=64, n_heads=64, n_idx_heads=64, d_idx=128, topk=512,
                          n_win=128, n_cap=32768, ctx=131072, seed=1))
# Pro-shaped CSA decode at 1M context: B=4, MXFP4 indexer keys and queries.
PRO_DECODE = _reg(Shape("pro_decode_1m", "csa_decode", "bf16", "mxfp4", B=4, T=1, m=4, c=512,
                        rope_dims=64, n_heads=128, n_idx_heads=64, d_idx=128, topk=1024,
                        n_win=128, n_cap=262144, ctx=1048576, seed=2))
# Flash-shaped chunked prefill: 8192 new tokens after a 57344-token prefix.
FLASH_PREFILL = _reg(Shape("flash_prefill_8k", "csa_prefill", "bf16", "bf16", B=1, T=8192, m=4,
                           c=512, rope_dims=64, n_heads=64, n_idx_heads=64, d_idx=128, topk=512,
                           n_win=128, n_cap=16384, ctx=57344, n_tok=8192, seed=3))
# HCA dense decode at 1M context: m'=128 -> 8192 entries, B=16.
HCA_DECODE = _reg(Shape("hca_decode_1m", "hca_decode", "bf16", "none", B=16, T=1, m=128,
                        c=512, rope_dims=64, n_heads=64, n_idx_heads=0, d_idx=0, topk=0,
                        n_win=128, n_cap=8192, ctx=1048576, seed=4, overlap=0))

# Mid-size parity cases: several tiles plus a ragged tail, ragged per-request contexts.
# Cache capacities are whole pages of 32 entries (128 tokens, the lcm(m, m') block of the
# paged cache); visibility inside them is ragged.
_reg(Shape("mid_decode_fp8", "csa_decode", "bf16", "fp8", B=3, T=1, m=4, c=512, rope_dims=64,
           n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128, n_cap=5024, ctx=19993,
           seed=11))
_reg(Shape("mid_decode_mxfp4", "csa_decode", "bf16", "mxfp4", B=3, T=1, m=4, c=512,
           rope_dims=64, n_heads=128, n_idx_heads=64, d_idx=128, topk=1024, n_win=128,
           n_cap=6016, ctx=23999, seed=12))
_reg(Shape("mid_decode_bf16", "csa_decode", "bf16", "bf16", B=2, T=1, m=4, c=512, rope_dims=64,
           n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128, n_cap=3008, ctx=12004,
           seed=13))
_reg(Shape("mid_prefill_bf16", "csa_prefill", "bf16", "bf16", B=1, T=384, m=4, c=512,
           rope_dims=64, n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128, n_cap=704,
           ctx=2416, n_tok=384, seed=14))
_reg(Shape("mid_hca_decode", "hca_decode", "bf16", "none", B=3, T=1, m=128, c=512, rope_dims=64,
           n_heads=64, n_idx_heads=0, d_idx=0, topk=0, n_win=128, n_cap=600, ctx=76900, seed=15,
           overlap=0))
# Few streams over a long dense list: each stream is split over many CTAs that each walk
# two or more chunks (the double-buffered 64-row form), with a ragged tail.
_reg(Shape("long_hca_decode", "hca_decode", "bf16", "none", B=2, T=1, m=128, c=512,
           rope_dims=64, n_heads=64, n_idx_heads=0, d_idx=0, topk=0, n_win=128, n_cap=4104,
           ctx=525389, seed=41, overlap=0))
# Degenerate decode cases: no visible entry (t < m), fewer visible entries than k,
# exactly k, and a cache shorter than floor(t/m). Also an MXFP4 one for the tensor-core
# indexer's edges (single partial tile, zero tiles, a request spanning many tiles).
_reg(Shape("edge_decode_bf16", "csa_decode", "bf16", "bf16", B=4, T=1, m=4, c=512, rope_dims=64,
           n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128, n_cap=608, ctx=0,
           seed=16, q_pos_override=(2, 37, 2051, 9999)))
_reg(Shape("edge_decode_mxfp4", "csa_decode", "bf16", "mxfp4", B=5, T=1, m=4, c=512,
           rope_dims=64, n_heads=128, n_idx_heads=64, d_idx=128, topk=1024, n_win=128,
           n_cap=4096, ctx=0, seed=18, q_pos_override=(3, 7, 515, 4099, 16384 + 77)))
_reg(Shape("edge_decode_mxfp4_long", "csa_decode", "bf16", "mxfp4", B=4, T=1, m=4, c=512,
           rope_dims=64, n_heads=128, n_idx_heads=64, d_idx=128, topk=1024, n_win=128,
           n_cap=16384, ctx=0, seed=19, q_pos_override=(4 * 16384 + 301, 48001, 13, 4100)))
# MXFP4 decode cases on the decode selector path (N_cap >= 8192): many CTAs per request,
# full visibility, exactly k and fewer than k visible entries, an empty request; and one
# with heavy ties (a request whose head weights are zero, one whose keys repeat).
_reg(Shape("mid_decode_mxfp4_sel", "csa_decode", "bf16", "mxfp4", B=6, T=1, m=4, c=512,
           rope_dims=64, n_heads=128, n_idx_heads=64, d_idx=128, topk=1024, n_win=128,
           n_cap=24576, ctx=0, seed=23,
           q_pos_override=(4 * 24576 + 3, 80007, 4 * 1024 + 2, 4 * 1023 + 1, 3, 20001)))
_reg(Shape("edge_decode_mxfp4_ties", "csa_decode", "bf16", "mxfp4", B=3, T=1, m=4, c=512,
           rope_dims=64, n_heads=128, n_idx_heads=64, d_idx=128, topk=1024, n_win=128,
           n_cap=12288, ctx=0, seed=24, q_pos_override=(4 * 12288, 4 * 12288 + 1, 30000),
           w_zero_requests=(0,), dup_keys=(1, 64)))
# Tensor-core indexer cases for fp8 and bf16 keys (cache capacity a multiple of 128): zero
# tiles, a single partial tile, several tiles, and more positions than the cache holds.
_reg(Shape("edge_decode_fp8_tc", "csa_decode", "bf16", "fp8", B=5, T=1, m=4, c=512,
           rope_dims=64, n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128,
           n_cap=4096, ctx=0, seed=20, q_pos_override=(3, 7, 515, 4099, 16384 + 77)))
_reg(Shape("edge_decode_bf16_tc", "csa_decode", "bf16", "bf16", B=4, T=1, m=4, c=512,
           rope_dims=64, n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128,
           n_cap=8192, ctx=0, seed=21, q_pos_override=(4 * 8192 + 301, 20001, 13, 4100)))
_reg(Shape("mid_prefill_bf16_tc", "csa_prefill", "bf16", "bf16", B=1, T=384, m=4, c=512,
           rope_dims=64, n_heads=64, n_idx_heads=64, d_idx=128, topk=512, n_win=128, n_cap=768,
           ctx=2416, n_tok=384, seed=22))
_reg(Shape("edge_hca_decode", "hca_decode", "bf16", "none", B=3, T=1, m=128, c=512, rope_dims=64,
           n_heads=64, n_idx_heads=0, d_idx=0, topk=0, n_win=128, n_cap=40, ctx=0, seed=17,
           overlap=0, q_pos_override=(0, 127, 9000)))
# Compression-only cases.
_reg(Shape("tiny_hca_compress", "hca_compress", "f32", "none", B=1, T=0, m=16, c=64, rope_dims=16,
           n_heads=0, n_idx_heads=0, d_idx=0, topk=0, n_win=0, n_cap=16, ctx=0, n_tok=256,
           seed=5, bias_std=0.1, overlap=0))
_reg(Shape("idx_key_compress", "csa_compress", "f32", "none", B=1, T=0, m=4, c=128, rope_dims=0,
           n_heads=0, n_idx_heads=0, d_idx=0, topk=0, n_win=0, n_cap=64, ctx=0, n_tok=256,
           seed=6, bias_std=0.1))


def sm_scale(s: Shape) -> float:
    """Attention logit scale used by every workload: 1/sqrt(c)."""
    return 1.0 / math.sqrt(s.c)


def decode_positions(s: Shape) -> np.ndarray:
    """Query positions [B, T] (int64).

    Decode: the new token after ``ctx`` cached tokens sits at position ctx. The mid-size
    cases give every request a different context (ragged visibility): request b uses
    ctx - 797*b (clamped at 0). Prefill: positions ctx .. ctx+T-1.
    """
    if s.kind in ("csa_decode", "hca_decode"):
        if s.q_pos_override:
            pos = np.array([[p] for p in s.q_pos_override], dtype=np.int64)
        elif s.name.startswith("mid_"):
            pos = np.array([[max(s.ctx - 797 * b, 0)] for b in range(s.B)], dtype=np.int64)
        else:
            pos = np.full((s.B, s.T), s.ctx, dtype=np.int64)
    else:
        pos = np.tile(np.arange(s.ctx, s.ctx + s.T, dtype=np.int64), (s.B, 1))
    return pos


def _normal(g, shape, std=1.0):
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _encode_io(x: np.ndarray, io: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if io == "bf16" else np.ascontiguousarray(x, np.float32)


def make_inputs(s: Shape, *, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw one workload's inputs. Returns host arrays (bf16 as uint16 bit patterns).

    Keys (present as the workload needs them):
      q [B,T,H,c], q_pos [B,T] int64, kv_cache [B,N_cap,c], win_kv [B,L_raw,c],
      win_pos0 [B] int64, sink [H] f32,
      qI [B,T,H_I,d_I] (f32 / bf16; MXFP4: qI packed [..,d_I/2] u8 + qI_scale [..,d_I/32] u8),
      KI [B,N_cap,d_I] (f32 / bf16; FP8: u8 codes + KI_scale [B,N_cap] f32; MXFP4: packed
      [..,d_I/2] + KI_scale [..,d_I/32] u8 in the blocked order of block_key_scales),
      w [B,T,H_I] f32,
      compression: Ca Cb Za Zb [n_tok,c], bias [2m,c] (rows 0..m-1 = B^a, m..2m-1 = B^b)
      (HCA: C, Z [n_tok,c], bias [m,c]); prev_Cb / prev_Zb [m,c] for a chunk that does not
      start the sequence. Also KI_f32 / qI_f32 (the fp32 draws before encoding) for the
      quantised indexer formats.
    """
    g = np.random.Generator(np.random.PCG64(s.seed if seed is None else seed))
    out: Dict[str, np.ndarray] = {}
    io = s.io
    B, T, H, c = s.B, s.T, s.n_heads, s.c
    out["q_pos"] = decode_positions(s)

    if s.kind in ("csa_compress", "hca_compress"):
        if s.overlap:
            for k in ("Ca", "Cb", "Za", "Zb"):
                out[k] = _encode_io(_normal(g, (s.n_tok, c)), io)
            out["bias"] = _encode_io(_normal(g, (2 * s.m, c), s.bias_std), io)
        else:
            for k in ("C", "Z"):
                out[k] = _encode_io(_normal(g, (s.n_tok, c)), io)
            out["bias"] = _encode_io(_normal(g, (s.m, c), s.bias_std), io)
        return out

    if s.kind == "csa_prefill":
        # listed first: per-token compression inputs and the bias
        for k in ("Ca", "Cb", "Za", "Zb"):
            out[k] = _encode_io(_normal(g, (s.n_tok, c)), io)
        out["bias"] = _encode_io(_normal(g, (2 * s.m, c), s.bias_std), io)
        if s.name.startswith("tiny"):
            out["q"] = _encode_io(_normal(g, (B, T, H, c)), io)
            out["qI"] = np.ascontiguousarray(_normal(g, (B, T, s.n_idx_heads, s.d_idx)))
            out["KI"] = np.ascontiguousarray(_normal(g, (B, s.n_cap, s.d_idx)))
            out["w"] = g.uniform(0.0, 1.0, size=(B, T, s.n_idx_heads)).astype(np.float32)
            win = _normal(g, (B, s.ctx + s.T, c))
            out["win_kv"] = _encode_io(win, io)
            out["win_pos0"] = np.zeros((B,), np.int64)
            out["kv_cache"] = np.zeros((B, s.n_cap, c), np.float32 if io == "f32" else np.uint16)
        else:
            qI = _normal(g, (B, T, s.n_idx_heads, s.d_idx))
            KI = _normal(g, (B, s.n_cap, s.d_idx))
            out["qI"], out["KI"] = f32_to_bf16_bits(qI), f32_to_bf16_bits(KI)
            out["w"] = _normal(g, (B, T, s.n_idx_heads))
            out["q"] = _encode_io(_normal(g, (B, T, H, c)), io)
            # extras: the cached prefix's compressed entries, the window's raw rows and the
            # state cache's uncompressed tail (last m tokens of the prefix, b-branch inputs)
            first = s.ctx // s.m
            kv = np.zeros((B, s.n_cap, c), np.uint16)
            kv[:, :first] = f32_to_bf16_bits(_normal(g, (B, first, c)))
            out["kv_cache"] = kv
            lo = max(s.ctx - s.n_win + 1, 0)
            out["win_kv"] = _encode_io(_normal(g, (B, s.ctx + s.T - lo, c)), io)
            out["win_pos0"] = np.full((B,), lo, np.int64)
            out["prev_Cb"] = _encode_io(_normal(g, (s.m, c)), io)
            out["prev_Zb"] = _encode_io(_normal(g, (s.m, c)), io)
        out["sink"] = (np.zeros((H,), np.float32) if s.sink == "zero"
                       else _normal(g, (H,)))
        return out

    # decode workloads (CSA and HCA): queries, the compressed cache, the window rows
    out["q"] = _encode_io(_normal(g, (B, T, H, c)), io)
    out["kv_cache"] = _encode_io(_normal(g, (B, s.n_cap, c)), io)
    # each request's window: n_win rows starting at max(t_b - n_win + 1, 0)
    out["win_kv"] = _encode_io(_normal(g, (B, s.n_win, c)), io)
    out["win_pos0"] = np.maximum(out["q_pos"][:, 0] - s.n_win + 1, 0).astype(np.int64)
    if s.kind == "csa_decode":
        qI = _normal(g, (B, T, s.n_idx_heads, s.d_idx))
        KI = _normal(g, (B, s.n_cap, s.d_idx))
        if s.dup_keys:
            rb, period = s.dup_keys
            KI[rb] = np.tile(KI[rb, :period], (s.n_cap // period, 1))
        if s.idx == "bf16":
            out["qI"], out["KI"] = f32_to_bf16_bits(qI), f32_to_bf16_bits(KI)
        elif s.idx == "fp8":
            out["qI"] = f32_to_bf16_bits(qI)
            out["KI"], out["KI_scale"] = quant_fp8_rowwise(KI)
            out["KI_f32"] = KI
        elif s.idx == "mxfp4":
            out["qI"], out["qI_scale"] = quant_mxfp4(qI)
            out["KI"], ks = quant_mxfp4(KI)
            out["KI_scale"] = block_key_scales(ks)
            out["KI_f32"], out["qI_f32"] = KI, qI
        else:
            raise ValueError(s.idx)
        out["w"] = _normal(g, (B, T, s.n_idx_heads))
        for rb in s.w_zero_requests:
            out["w"][rb] = 0.0
    out["sink"] = _normal(g, (H,))
    return out


def params_of(s: Shape) -> Dict[str, float]:
    """Method constants of a workload as a plain dict (what the library's csa_params holds)."""
    return dict(m=s.m, overlap=s.overlap, c=s.c, rope_dims=s.rope_dims, rope_base=s.rope_base,
                rms_eps=s.rms_eps, sm_scale=sm_scale(s), n_heads=s.n_heads,
                n_idx_heads=s.n_idx_heads, d_idx=s.d_idx, topk=s.topk, n_win=s.n_win)


def make_state_stream(*, B: int, n_tok: int, m: int, c: int, overlap: int, io: str,
                      seed: int) -> Dict[str, np.ndarray]:
    """Seeded raw token rows for decode-time appends to a state cache: for every request
    b < B the rows of tokens 0 .. n_tok-1 (a request resumed at position t0 takes the
    rows before t0 as its prefill), drawn ~N(0,1) in the order Ca, Cb, Za, Zb (CSA; C, Z
    for HCA), then the window rows, then the pooling bias ([2m, c] CSA, [m, c] HCA; std
    1), each [B, n_tok, c]; encoded as ``io`` ("f32" or "bf16" bit patterns). The shapes
    follow the models' c = 512, m = 4 / m' = 128 [【论文解读】DeepSeek-V4 三、预训练 (二)]."""
    g = np.random.default_rng(seed)
    names = ("Ca", "Cb", "Za", "Zb") if overlap else ("Ca", "Za")
    out = {k: _encode_io(_normal(g, (B, n_tok, c)), io) for k in names}
    out["win"] = _encode_io(_normal(g, (B, n_tok, c)), io)
    out["bias"] = _encode_io(_normal(g, ((2 if overlap else 1) * m, c)), io)
    return out


def make_out_proj_inputs(*, Q: int, H: int, c: int, g: int, d_g: int, d: int,
                         seed: int) -> Dict[str, np.ndarray]:
    """Seeded inputs of the grouped output projection, as bf16 bit patterns: the attention
    outputs o [Q, H*c] ~ N(0,1), then the group matrices w_grp [g, c*H/g, d_g] and the
    output matrix w_out [g*d_g, d], each ~N(0, 1/rows) (random initialisation that keeps
    the sums O(1)). Shapes of 【论文解读】DeepSeek-V4 三、预训练 (二): g = 8 / 16,
    d_g = 1024, d = 4096 / 7168."""
    g_ = np.random.default_rng(seed)
    k1 = c * (H // g)
    o = _normal(g_, (Q, H * c))
    w_grp = _normal(g_, (g, k1, d_g), std=1.0 / math.sqrt(k1))
    w_out = _normal(g_, (g * d_g, d), std=1.0 / math.sqrt(g * d_g))
    return {"o": f32_to_bf16_bits(o), "w_grp": f32_to_bf16_bits(w_grp),
            "w_out": f32_to_bf16_bits(w_out)}

