// Host build of the state-append arithmetic (csrc/state_append.cuh) for the CPU tests: the
// same __host__ __device__ functions the kernel calls, run request by request and channel
// by channel in the kernel's order, on host arrays. Every offset written is checked against
// the buffer sizes first. Test infrastructure: the library never links it.
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <vector>

#include "state_append.cuh"

namespace {

using namespace csa::state;

// One finished row `fin` [c] stored at page row `prow` in the chosen format; returns a
// negative code if an offset would fall outside its buffer.
int store_row(const Args& a, const std::vector<float>& fin, size_t prow, size_t page_bytes,
              size_t scale_bytes) {
  const int c = a.c;
  if (a.out == kOutMixed) {
    const int r0 = c - a.rope_dims;
    const size_t rb = (size_t)(c + a.rope_dims);
    if ((prow + 1) * rb > page_bytes || (prow + 1) * sizeof(float) > scale_bytes) return -16;
    float amax = 0.f;
    for (int j = 0; j < r0; ++j) amax = fmaxf(amax, fabsf(fin[j]));
    const float scale = fp8_row_scale(amax);
    uint8_t* rowp = static_cast<uint8_t*>(a.pages) + prow * rb;
    __nv_bfloat16* rope = reinterpret_cast<__nv_bfloat16*>(rowp + r0);
    for (int j = 0; j < c; ++j) {
      if (j < r0) rowp[j] = (uint8_t)fp8_code(fin[j], scale);
      else rope[j - r0] = __float2bfloat16_rn(fin[j]);
    }
    static_cast<float*>(a.page_scales)[prow] = scale;
    return 0;
  }
  if (a.out == kOutFp8) {
    if ((prow + 1) * c > page_bytes || (prow + 1) * sizeof(float) > scale_bytes) return -13;
    float amax = 0.f;
    for (int j = 0; j < c; ++j) amax = fmaxf(amax, fabsf(fin[j]));
    const float scale = fp8_row_scale(amax);
    uint8_t* codes = static_cast<uint8_t*>(a.pages) + prow * c;
    for (int j = 0; j < c; ++j) codes[j] = (uint8_t)fp8_code(fin[j], scale);
    static_cast<float*>(a.page_scales)[prow] = scale;
    return 0;
  }
  // MXFP4
  if ((prow + 1) * (c / 2) > page_bytes) return -14;
  uint8_t* packed = static_cast<uint8_t*>(a.pages) + prow * (c / 2);
  uint8_t* exps = static_cast<uint8_t*>(a.page_scales);
  const int slot = (int)(prow % (size_t)a.page_rows);
  for (int blk = 0; blk < c / 32; ++blk) {
    float amax = 0.f;
    for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(fin[32 * blk + k]));
    const int E = mx_exponent(amax);
    for (int k = 0; k < 32; k += 2) {
      const int j = 32 * blk + k;
      const uint32_t lo = e2m1_code(fin[j] / pow2f(E)), hi = e2m1_code(fin[j + 1] / pow2f(E));
      packed[j >> 1] = (uint8_t)(lo | (hi << 4));
    }
    const size_t so = mx_scale_offset(prow - slot, slot, blk);
    if (so >= scale_bytes) return -15;
    exps[so] = (uint8_t)(E + 127);
  }
  return 0;
}

template <typename T>
int run(Args a, int32_t* status, size_t state_elems, size_t ring_elems, size_t page_bytes,
        size_t scale_bytes) {
  std::vector<float> row(a.c), fin(a.c);
  for (int b = 0; b < a.B; ++b) {
    const int64_t t = a.pos[b];
    int64_t i = 0;
    size_t off = 0;
    const int s = append_status(a, b, t, &i, &off);
    status[b] = s;
    if (s < 0) continue;
    for (int j = 0; j < a.c; ++j) {
      for (int r = 0; r < rows(a); ++r)
        if (state_index(a, b, t, r, j) >= state_elems) return -10;
      if (a.win_ring && ((size_t)b * a.n_win + (size_t)(t % a.n_win)) * a.c + j >= ring_elems)
        return -11;
      store_channel<T>(a, b, t, j);
    }
    if (s == kAppendOnly) continue;
    float ss = 0.f;
    for (int j = 0; j < a.c; ++j) {
      row[j] = pool_channel<T>(a, b, i, j);
      ss = fmaf(row[j], row[j], ss);
    }
    const float rstd = a.finalize ? 1.f / sqrtf(ss / (float)a.c + a.eps) : 1.f;
    for (int j = 0; j < a.c; ++j)
      fin[j] = a.finalize ? final_channel<T>(a, row.data(), rstd, i, j) : row[j];
    if (a.out == kOutIo) {
      if ((off + a.c) * sizeof(T) > page_bytes) return -12;
      T* out = static_cast<T*>(a.pages) + off;
      for (int j = 0; j < a.c; ++j) st(out, j, fin[j]);
      continue;
    }
    const int rc = store_row(a, fin, off / (size_t)a.c, page_bytes, scale_bytes);
    if (rc != 0) return rc;
  }
  return 0;
}

}  // namespace

// out: 0 = io dtype, 1 = FP8 rows, 2 = MXFP4 rows, 3 = mixed FP8 / bf16 rows;
// page_bytes / scale_bytes: buffer sizes.
extern "C" int state_append_host(int bf16, int B, int m, int c, int overlap, int rope_dims,
                                 double rope_base, int finalize, int n_win, int n_pages,
                                 int page_rows, int max_pages, float eps, int out,
                                 const int64_t* pos, const void* Ca, const void* Cb,
                                 const void* Za, const void* Zb, const void* win_row,
                                 const void* bias, const void* rms_w, void* state,
                                 void* win_ring, void* pages, size_t page_bytes,
                                 void* page_scales, size_t scale_bytes,
                                 const int32_t* page_table, int32_t* status) {
  Args a{};
  a.B = B; a.m = m; a.c = c; a.overlap = overlap; a.rope_dims = rope_dims;
  a.finalize = finalize; a.n_win = n_win; a.n_pages = n_pages; a.page_rows = page_rows;
  a.max_pages = max_pages; a.eps = eps; a.out = out; a.pos = pos; a.Ca = Ca; a.Cb = Cb;
  a.Za = Za; a.Zb = Zb; a.win_row = win_row; a.bias = bias; a.rms_w = rms_w; a.state = state;
  a.win_ring = win_ring; a.pages = pages; a.page_scales = page_scales;
  a.page_table = page_table;
  for (int p = 0; p < rope_dims / 2; ++p)
    a.inv_freq[p] = std::exp2(-2.0 * p / rope_dims * std::log2(rope_base));
  const size_t state_elems = (size_t)B * (overlap ? 2 * m : m) * (overlap ? 4 : 2) * c;
  const size_t ring_elems = (size_t)B * (n_win > 0 ? n_win : 0) * c;
  return bf16 ? run<__nv_bfloat16>(a, status, state_elems, ring_elems, page_bytes, scale_bytes)
              : run<float>(a, status, state_elems, ring_elems, page_bytes, scale_bytes);
}

// The row encoders alone: rows [n, c] fp32 -> FP8 (out = 1: codes [n, c], scales [n] fp32)
// or MXFP4 (out = 2: packed [n, c/2], exponents [n, 4] in the 128-row blocked layout;
// n a multiple of 128, c = 128).
extern "C" int encode_rows_host(int out, int n, int c, const float* rows, void* codes,
                                void* scales) {
  Args a{};
  a.c = c; a.out = out; a.page_rows = n; a.pages = codes; a.page_scales = scales;
  std::vector<float> fin(c);
  const size_t page_bytes = out == kOutFp8 ? (size_t)n * c : (size_t)n * c / 2;
  const size_t scale_bytes = out == kOutFp8 ? (size_t)n * sizeof(float) : (size_t)n * 4;
  for (int r = 0; r < n; ++r) {
    for (int j = 0; j < c; ++j) fin[j] = rows[(size_t)r * c + j];
    const int rc = store_row(a, fin, (size_t)r, page_bytes, scale_bytes);
    if (rc != 0) return rc;
  }
  return 0;
}

// csa_state_resume's arithmetic: the chunk's last raw rows and window rows into the state.
extern "C" int state_resume_host(int bf16, int B, int m, int c, int overlap, int n_win,
                                 int64_t first_tok, int64_t n_tok, const void* Ca, const void* Cb,
                                 const void* Za, const void* Zb, const void* win_rows,
                                 void* state, void* win_ring) {
  Args a{};
  a.B = B; a.m = m; a.c = c; a.overlap = overlap; a.n_win = n_win; a.Ca = Ca; a.Cb = Cb;
  a.Za = Za; a.Zb = Zb; a.win_row = win_rows; a.state = state; a.win_ring = win_ring;
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < c; ++j)
      bf16 ? resume_channel<__nv_bfloat16>(a, b, first_tok, n_tok, j)
           : resume_channel<float>(a, b, first_tok, n_tok, j);
  return 0;
}

// csa_encode_paged's arithmetic: rows [B, n, c] (io dtype) = entries first_entry .. of every
// request, stored through the page table in the format `out` (0 io, 1 FP8, 2 MXFP4, 3 mixed);
// status[b * n + i] = the entry's status (1 stored, < 0 skipped).
extern "C" int encode_paged_host(int bf16, int B, int64_t n, int64_t first_entry, int c,
                                 int rope_dims, int out, int n_pages, int page_rows,
                                 int max_pages, const void* rows, void* pages,
                                 size_t page_bytes, void* page_scales, size_t scale_bytes,
                                 const int32_t* page_table, int32_t* status) {
  Args a{};
  a.B = B; a.c = c; a.rope_dims = rope_dims; a.out = out; a.n_pages = n_pages;
  a.page_rows = page_rows; a.max_pages = max_pages; a.pages = pages;
  a.page_scales = page_scales; a.page_table = page_table;
  std::vector<float> fin(c);
  for (int b = 0; b < B; ++b)
    for (int64_t i = 0; i < n; ++i) {
      size_t off = 0;
      const int s = entry_offset(a, b, first_entry + i, &off);
      status[(size_t)b * n + i] = s;
      if (s != kCompress) continue;
      for (int j = 0; j < c; ++j) {
        const size_t k = ((size_t)b * n + i) * c + j;
        fin[j] = bf16 ? ld(static_cast<const __nv_bfloat16*>(rows), k)
                      : ld(static_cast<const float*>(rows), k);
      }
      if (out == kOutIo) {
        if ((off + c) * (bf16 ? 2 : 4) > page_bytes) return -12;
        for (int j = 0; j < c; ++j) {
          if (bf16) st(static_cast<__nv_bfloat16*>(pages) + off, j, fin[j]);
          else st(static_cast<float*>(pages) + off, j, fin[j]);
        }
        continue;
      }
      const int rc = store_row(a, fin, off / (size_t)c, page_bytes, scale_bytes);
      if (rc != 0) return rc;
    }
  return 0;
}
