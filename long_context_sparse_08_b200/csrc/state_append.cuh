// Decode-time compression with a state cache: the index arithmetic and the per-channel
// math of appending one token to one request, written once as __host__ __device__
// functions. The kernel (state_append.cu) runs them with a CTA per request and threads
// over channels; a host build of the same functions lets the CPU tests check slots, pages
// and values without a GPU.
//
// 【论文解读】DeepSeek-V4, 二、基础设施 (六) 推理框架: a state cache holds the sliding
// window and the raw tail tokens of a compression block not yet full; finished entries go
// to a paged cache whose blocks cover a multiple of lcm(m, m') raw tokens.
// 一(三)1(1) / 2(1): the compression of a block; 3(1), 3(2): RMSNorm and RoPE of an entry.
//
// State layout of request b ([B, S, R, c], io dtype): token p lives in slot p mod S, row r
// of the slot is one of its raw tensors. CSA (overlap): S = 2m, rows Ca, Za, Cb, Zb -- the
// 2m slots hold the open block (its a- and b-rows) and the previous block (whose b-rows
// entry i reads). HCA: S = m', rows C, Z.
//
// Finished rows are stored in the io dtype, or in the formats the indexers read (the
// compressed indexer keys are one of the caches a decode step extends):
//   FP8: e4m3 codes [page_rows, c] per page, one fp32 scale per row (amax / 448);
//   MXFP4 (c = 128): e2m1 pairs [page_rows, 64] per page (element 2j in the low nibble),
//     one e8m0 exponent per 32 elements (OCP MX v1.0: floor(log2 amax) - 2), stored per block
//     of 128 rows with byte 16*i + 4*j + b holding exponent b of row 32*j + i.
// and the KV entries in the mixed precision of 一(三)4 item 1:
//   mixed: c + r bytes per row, the e4m3 codes of the first c-r values (one fp32 row scale,
//     amax of those values / 448) then the last r (RoPE) values as bf16.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

namespace csa {
namespace state {

#define CSA_HD __host__ __device__ __forceinline__

enum { kRowCa = 0, kRowZa = 1, kRowCb = 2, kRowZb = 3 };  // HCA: C = row 0, Z = row 1

// Status of one request's append (uniform over the CTA).
enum {
  kAppendOnly = 0,   // the token does not finish a block
  kCompress = 1,     // the token finishes entry i: compress it into its page
  kErrPosition = -1, // negative position
  kErrPageSlot = -2, // entry's logical page beyond the page table
  kErrPageId = -3    // page table entry outside [0, n_pages)
};

enum { kOutIo = 0, kOutFp8 = 1, kOutMxfp4 = 2, kOutMixed = 3 };  // storage of finished rows

struct Args {
  int B, m, c, overlap, rope_dims, finalize, n_win, n_pages, page_rows, max_pages, out;
  float eps;
  const int64_t* pos;  // [B] position of each request's new token
  const void *Ca, *Cb, *Za, *Zb, *win_row, *bias, *rms_w;  // new rows [B, c]; bias; gamma
  void *state, *win_ring, *pages, *page_scales;
  const int32_t* page_table;  // [B, max_pages]
  double inv_freq[256];       // RoPE pair frequencies base^(-2p/r), p < r/2
};

CSA_HD float ld(const float* p, size_t i) { return p[i]; }
CSA_HD float ld(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
CSA_HD void st(float* p, size_t i, float v) { p[i] = v; }
CSA_HD void st(__nv_bfloat16* p, size_t i, float v) { p[i] = __float2bfloat16_rn(v); }

CSA_HD int slots(const Args& a) { return a.overlap ? 2 * a.m : a.m; }
CSA_HD int rows(const Args& a) { return a.overlap ? 4 : 2; }

// element (request b, state slot, raw tensor r, channel j) of the state
CSA_HD size_t slot_index(const Args& a, int64_t b, int slot, int r, int j) {
  return (((size_t)b * slots(a) + (size_t)slot) * rows(a) + r) * (size_t)a.c + j;
}
// element (request b, token p, raw tensor r, channel j) of the state: token p in slot p mod S
CSA_HD size_t state_index(const Args& a, int64_t b, int64_t p, int r, int j) {
  return slot_index(a, b, (int)(p % slots(a)), r, j);
}

// Element offset in `pages` of the row of entry i of request b, through the page table:
// kCompress, or kErrPageSlot / kErrPageId when the entry has no valid page.
CSA_HD int entry_offset(const Args& a, int64_t b, int64_t i, size_t* out_off) {
  const int64_t pg = i / a.page_rows;
  if (pg >= a.max_pages) return kErrPageSlot;
  const int32_t page = a.page_table[(size_t)b * a.max_pages + pg];
  if (page < 0 || page >= a.n_pages) return kErrPageId;
  *out_off = ((size_t)page * a.page_rows + (size_t)(i % a.page_rows)) * (size_t)a.c;
  return kCompress;
}

// What the token at position t of request b does; for kCompress also the entry index and
// the element offset of its row in `pages`.
CSA_HD int append_status(const Args& a, int64_t b, int64_t t, int64_t* entry, size_t* out_off) {
  if (t < 0) return kErrPosition;
  if ((t + 1) % a.m != 0) return kAppendOnly;
  const int64_t i = t / a.m;
  const int s = entry_offset(a, b, i, out_off);
  if (s == kCompress) *entry = i;
  return s;
}

// Channel j of the new token: raw rows into the state, window row into the ring.
template <typename T>
CSA_HD void store_channel(const Args& a, int64_t b, int64_t t, int j) {
  T* s = static_cast<T*>(a.state);
  const size_t src = (size_t)b * a.c + j;
  st(s, state_index(a, b, t, kRowCa, j), ld(static_cast<const T*>(a.Ca), src));
  st(s, state_index(a, b, t, kRowZa, j), ld(static_cast<const T*>(a.Za), src));
  if (a.overlap) {
    st(s, state_index(a, b, t, kRowCb, j), ld(static_cast<const T*>(a.Cb), src));
    st(s, state_index(a, b, t, kRowZb, j), ld(static_cast<const T*>(a.Zb), src));
  }
  if (a.win_ring != nullptr) {
    const size_t dst = ((size_t)b * a.n_win + (size_t)(t % a.n_win)) * a.c + j;
    st(static_cast<T*>(a.win_ring), dst, ld(static_cast<const T*>(a.win_row), src));
  }
}

// Channel j of a request resumed after a prefill chunk of tokens first_tok .. first_tok +
// n_tok - 1 (rows [B, n_tok, c] in a.Ca / a.Za / a.Cb / a.Zb and a.win_row): the chunk's last
// raw rows into their state slots, its last window rows into the ring, by absolute position.
template <typename T>
CSA_HD void resume_channel(const Args& a, int64_t b, int64_t first_tok, int64_t n_tok, int j) {
  T* s = static_cast<T*>(a.state);
  const int S = slots(a);
  // the slot (and ring row) of a token advance by one per token: one modulo per loop
  const int64_t t0 = n_tok > S ? n_tok - S : 0;
  int slot = (int)((first_tok + t0) % S);
  for (int64_t t = t0; t < n_tok; ++t) {
    const size_t src = ((size_t)b * n_tok + t) * a.c + j;
    st(s, slot_index(a, b, slot, kRowCa, j), ld(static_cast<const T*>(a.Ca), src));
    st(s, slot_index(a, b, slot, kRowZa, j), ld(static_cast<const T*>(a.Za), src));
    if (a.overlap) {
      st(s, slot_index(a, b, slot, kRowCb, j), ld(static_cast<const T*>(a.Cb), src));
      st(s, slot_index(a, b, slot, kRowZb, j), ld(static_cast<const T*>(a.Zb), src));
    }
    slot = slot + 1 == S ? 0 : slot + 1;
  }
  if (a.win_ring != nullptr) {
    const int64_t w0 = n_tok > a.n_win ? n_tok - a.n_win : 0;
    int row = (int)((first_tok + w0) % a.n_win);
    for (int64_t t = w0; t < n_tok; ++t) {
      const size_t src = ((size_t)b * n_tok + t) * a.c + j;
      const size_t dst = ((size_t)b * a.n_win + (size_t)row) * a.c + j;
      st(static_cast<T*>(a.win_ring), dst, ld(static_cast<const T*>(a.win_row), src));
      row = row + 1 == a.n_win ? 0 : row + 1;
    }
  }
}

// Channel j of entry i, pooled from the state: softmax over the block's logits plus biases
// (CSA: the a-rows of block i, and for i > 0 the b-rows of block i-1), weighted sum of the
// values. Same operation order as the whole-chunk compression kernel.
template <typename T>
CSA_HD float pool_channel(const Args& a, int64_t b, int64_t i, int j) {
  const T* s = static_cast<const T*>(a.state);
  const T* bias = static_cast<const T*>(a.bias);
  const int m = a.m;
  const bool has_b = a.overlap && i > 0;
  float mx = -INFINITY;
  for (int r = 0; r < m; ++r)
    mx = fmaxf(mx, ld(s, state_index(a, b, m * i + r, kRowZa, j)) + ld(bias, (size_t)r * a.c + j));
  if (has_b)
    for (int r = 0; r < m; ++r)
      mx = fmaxf(mx, ld(s, state_index(a, b, m * (i - 1) + r, kRowZb, j)) +
                         ld(bias, (size_t)(m + r) * a.c + j));
  float den = 0.f, num = 0.f;
  for (int r = 0; r < m; ++r) {
    const int64_t p = m * i + r;
    const float e = expf(ld(s, state_index(a, b, p, kRowZa, j)) + ld(bias, (size_t)r * a.c + j) - mx);
    den += e;
    num = fmaf(e, ld(s, state_index(a, b, p, kRowCa, j)), num);
  }
  if (has_b)
    for (int r = 0; r < m; ++r) {
      const int64_t p = m * (i - 1) + r;
      const float e = expf(ld(s, state_index(a, b, p, kRowZb, j)) +
                           ld(bias, (size_t)(m + r) * a.c + j) - mx);
      den += e;
      num = fmaf(e, ld(s, state_index(a, b, p, kRowCb, j)), num);
    }
  return num / den;
}

// cos / sin of pos * inv_freq: the angle (up to ~1e6 rad) is reduced modulo 2*pi in double
// with a two-part 2*pi, then evaluated in fp32.
CSA_HD void rope_cs(double pos, double inv_freq, float* cs, float* sn) {
  const double x = pos * inv_freq;
  const double k = rint(x * 0.15915494309189535);  // x / (2*pi)
  double red = fma(-k, 6.283185307179586232, x);
  red = fma(-k, 2.4492935982947064e-16, red);
  sincosf((float)red, sn, cs);
}

// Channel j of the finished row: RMSNorm (rstd = 1/sqrt(mean(x^2) + eps), weight gamma),
// then RoPE at position m*i on the last r dims (pairs (2p, 2p+1) of that slice).
template <typename T>
CSA_HD float final_channel(const Args& a, const float* row, float rstd, int64_t i, int j) {
  const T* g = static_cast<const T*>(a.rms_w);
  float v = row[j] * rstd * (g ? ld(g, j) : 1.f);
  const int r0 = a.c - a.rope_dims;
  if (j >= r0) {
    const int partner = j ^ 1;  // r0 is even
    const float u = row[partner] * rstd * (g ? ld(g, partner) : 1.f);
    float cs, sn;
    rope_cs((double)a.m * (double)i, a.inv_freq[(j - r0) >> 1], &cs, &sn);
    v = ((j - r0) & 1) == 0 ? v * cs - u * sn : u * sn + v * cs;
  }
  return v;
}

// ---- storage formats of finished rows (the same encodings the input generators use) ----

// e4m3 code of v: nearest value, ties to even, saturating at +-448 (CUDA's conversion).
CSA_HD uint32_t e4m3_code(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Row scale of the FP8 format: amax / 448 in fp32 (0 for an all-zero row, whose codes are 0).
CSA_HD float fp8_row_scale(float amax) { return amax / 448.f; }
CSA_HD uint32_t fp8_code(float v, float scale) {
  return e4m3_code(v / (scale > 0.f ? scale : 1.f));
}

// Shared exponent of a 32-element MX block with largest magnitude amax: floor(log2 amax) - 2
// (2 is e2m1's largest exponent), clamped to e8m0's [-127, 127]; -127 for a zero block.
CSA_HD int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  int e = 0;
  frexpf(amax, &e);  // amax = f * 2^e with f in [0.5, 1): floor(log2 amax) = e - 1
  const int E = e - 1 - 2;
  return E < -127 ? -127 : (E > 127 ? 127 : E);
}

// 2^E as a float (E = -127 is a subnormal).
CSA_HD float pow2f(int E) {
  const uint32_t u = E >= -126 ? (uint32_t)(E + 127) << 23 : 0x00400000u;
  float f;
  memcpy(&f, &u, sizeof(f));
  return f;
}

// e2m1 code of v (already divided by its block's 2^E): the nearest magnitude of
// {0, .5, 1, 1.5, 2, 3, 4, 6} (at a midpoint the even code), saturating at 6; bit 3 is the
// sign of a negative value with a nonzero magnitude.
CSA_HD uint32_t e2m1_code(float v) {
  const float a = fminf(fabsf(v), 6.f);
  const float mids[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.f};
  uint32_t code = 0;
  for (int k = 0; k < 7; ++k) code += a > mids[k] ? 1u : 0u;
  for (int k = 1; k < 7; k += 2)
    if (a == mids[k]) code = (uint32_t)k + 1;  // midpoint above an odd code: round up
  return (v < 0.f && code > 0) ? (code | 8u) : code;
}

// Byte offset, in a page's MXFP4 exponents, of exponent b of page row `row`: rows are
// stored in blocks of 128 with byte 16*i + 4*j + b holding exponent b of row 32*j + i.
CSA_HD size_t mx_scale_offset(size_t page_row0, int row, int b) {
  const int blk = row / 128, kk = row % 128;
  return (page_row0 + (size_t)blk * 128) * 4 + (size_t)(16 * (kk % 32) + 4 * (kk / 32) + b);
}

#undef CSA_HD

}  // namespace state
}  // namespace csa
