// Decode-time compression with a state cache: append one token per request.
//
// 【论文解读】DeepSeek-V4, 二、基础设施 (六) 推理框架 (state cache of the window and the
// unfinished compression tail; paged cache of finished entries) and DeepseekV4论文解析,
// 2. Hybrid Attention：CSA + HCA, 从注意力公式到可部署系统 (a logical block of
// lcm(4, 128) = 128 raw tokens is 32 CSA entries or 1 HCA entry).
//
// One CTA per request, threads over channels. Every thread stores its channels of the new
// token (raw rows into the state slot, window row into the ring); when the token finishes
// a block, each thread pools its channels of the entry from the state (it reads back only
// what it or earlier launches wrote), the CTA reduces the sum of squares for the RMSNorm,
// and the rotated row goes to its page. Work per request is a few KB: the kernel is
// launch-latency bound, and one launch serves the whole decode batch.
#include "common.cuh"
#include "internal.h"
#include "state_append.cuh"

namespace csa {

namespace {

// device-side error word of this translation unit (0 = none; the first code wins)
__device__ int g_state_error = 0;

enum { kErrBase = 320 };  // stored code = kErrBase - status (321 position, 322 page slot, 323 page id)
enum { kErrEncodeBase = 322 };  // csa_encode_paged: 324 page slot, 325 page id

// Block-wide max of non-negative values; `red` is shared scratch of >= 32 floats.
__device__ __forceinline__ float block_max_nonneg(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.f;
  if (wid == 0) t = warp_max(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

// The finished row fin[c] (this thread's channels j = threadIdx.x + k*blockDim.x written by
// this thread; amax = this thread's max |fin[j]|) stored at element offset `off` of `pages`
// in the format a.out. Every thread of the CTA calls it (block reductions inside).
template <typename T>
__device__ __forceinline__ void store_finished(const state::Args& a, const float* fin,
                                               float amax, size_t off, float* red) {
  if (a.out == state::kOutIo) {
    T* out = static_cast<T*>(a.pages) + off;
    for (int j = threadIdx.x; j < a.c; j += blockDim.x) state::st(out, j, fin[j]);
    return;
  }
  const size_t prow = off / (size_t)a.c;  // global row index in the pages
  if (a.out == state::kOutMixed) {
    // e4m3 for the first c - r values (their own amax), bf16 for the RoPE values
    const int r0 = a.c - a.rope_dims;
    float am = 0.f;
    for (int j = threadIdx.x; j < r0; j += blockDim.x) am = fmaxf(am, fabsf(fin[j]));
    const float scale = state::fp8_row_scale(block_max_nonneg(am, red));
    uint8_t* rowp = static_cast<uint8_t*>(a.pages) + prow * (size_t)(a.c + a.rope_dims);
    __nv_bfloat16* rope = reinterpret_cast<__nv_bfloat16*>(rowp + r0);
    for (int j = threadIdx.x; j < a.c; j += blockDim.x) {
      if (j < r0) rowp[j] = (uint8_t)state::fp8_code(fin[j], scale);
      else rope[j - r0] = __float2bfloat16_rn(fin[j]);
    }
    if (threadIdx.x == 0) static_cast<float*>(a.page_scales)[prow] = scale;
    return;
  }
  if (a.out == state::kOutFp8) {
    const float scale = state::fp8_row_scale(block_max_nonneg(amax, red));
    uint8_t* codes = static_cast<uint8_t*>(a.pages) + off;
    for (int j = threadIdx.x; j < a.c; j += blockDim.x)
      codes[j] = (uint8_t)state::fp8_code(fin[j], scale);
    if (threadIdx.x == 0) static_cast<float*>(a.page_scales)[prow] = scale;
    return;
  }
  // MXFP4: a warp's 32 consecutive channels are one MX block (c and blockDim are multiples
  // of 32, so a warp's lanes are all in or all out of the loop)
  uint8_t* packed = static_cast<uint8_t*>(a.pages) + off / 2;
  uint8_t* exps = static_cast<uint8_t*>(a.page_scales);
  const int slot = (int)(prow % (size_t)a.page_rows);
  for (int j = threadIdx.x; j < a.c; j += blockDim.x) {
    const float v = fin[j];
    const int E = state::mx_exponent(warp_max(fabsf(v)));
    const uint32_t code = state::e2m1_code(v / state::pow2f(E));
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, code, 1);
    if ((j & 1) == 0) packed[j >> 1] = (uint8_t)(code | (hi << 4));
    if ((j & 31) == 0) exps[state::mx_scale_offset(prow - slot, slot, j >> 5)] = (uint8_t)(E + 127);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_state_append(state::Args a) {
  extern __shared__ float row[];  // [2c]: pooled row, then the finished row
  __shared__ float red[32];
  float* fin = row + a.c;
  const int b = blockIdx.x;
  const int64_t t = a.pos[b];
  int64_t i = 0;
  size_t off = 0;
  const int s = state::append_status(a, b, t, &i, &off);  // the same in every thread
  if (s < 0) {
    if (threadIdx.x == 0) atomicCAS(&g_state_error, 0, kErrBase - s);
    return;
  }
  for (int j = threadIdx.x; j < a.c; j += blockDim.x) state::store_channel<T>(a, b, t, j);
  if (s == state::kAppendOnly) return;
  float ss = 0.f;
  for (int j = threadIdx.x; j < a.c; j += blockDim.x) {
    const float v = state::pool_channel<T>(a, b, i, j);
    row[j] = v;
    ss = fmaf(v, v, ss);
  }
  float rstd = 1.f;
  if (a.finalize) {
    const float tot = block_sum(ss, red);  // also orders the row[] writes before the reads
    rstd = rsqrtf(tot / (float)a.c + a.eps);
  }
  float amax = 0.f;
  for (int j = threadIdx.x; j < a.c; j += blockDim.x) {
    const float v = a.finalize ? state::final_channel<T>(a, row, rstd, i, j) : row[j];
    fin[j] = v;  // read back by this thread only
    amax = fmaxf(amax, fabsf(v));
  }
  store_finished<T>(a, fin, amax, off, red);
}

template <typename T>
__global__ void __launch_bounds__(256) k_state_resume(state::Args a, int64_t first_tok,
                                                      int64_t n_tok) {
  for (int j = threadIdx.x; j < a.c; j += blockDim.x)
    state::resume_channel<T>(a, blockIdx.x, first_tok, n_tok, j);
}

// csa_encode_paged: entry first_entry + blockIdx.x of request blockIdx.y, given in the io
// dtype (rows [B, n, c]), stored into its page in the format a.out exactly as
// k_state_append stores a finished row.
template <typename T>
__global__ void __launch_bounds__(256) k_encode_paged(state::Args a, const void* rows,
                                                      int64_t n, int64_t first_entry) {
  extern __shared__ float fin[];  // [c]
  __shared__ float red[32];
  const int b = blockIdx.y;
  size_t off = 0;
  const int s = state::entry_offset(a, b, first_entry + blockIdx.x, &off);  // CTA-uniform
  if (s != state::kCompress) {
    if (threadIdx.x == 0) atomicCAS(&g_state_error, 0, kErrEncodeBase - s);
    return;
  }
  const T* src = static_cast<const T*>(rows) + ((size_t)b * n + blockIdx.x) * (size_t)a.c;
  float amax = 0.f;
  for (int j = threadIdx.x; j < a.c; j += blockDim.x) {
    const float v = state::ld(src, (size_t)j);
    fin[j] = v;  // read back by this thread only
    amax = fmaxf(amax, fabsf(v));
  }
  store_finished<T>(a, fin, amax, off, red);
}

}  // namespace

cudaError_t launch_state_resume(const state::Args& a, bool bf16, int64_t first_tok,
                                int64_t n_tok, cudaStream_t st) {
  if (a.B == 0 || n_tok == 0) return cudaSuccess;
  const int threads = a.c >= 256 ? 256 : ((a.c + 31) / 32) * 32;
  cudaError_t e = bf16 ? launch(false, k_state_resume<__nv_bfloat16>, dim3(a.B), dim3(threads), 0,
                                st, a, first_tok, n_tok)
                       : launch(false, k_state_resume<float>, dim3(a.B), dim3(threads), 0, st, a,
                                first_tok, n_tok);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_state_append(const state::Args& a, bool bf16, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  const int threads = a.c >= 256 ? 256 : ((a.c + 31) / 32) * 32;
  const size_t smem = 2 * (size_t)a.c * sizeof(float);
  cudaError_t e = bf16 ? launch(false, k_state_append<__nv_bfloat16>, dim3(a.B), dim3(threads),
                                smem, st, a)
                       : launch(false, k_state_append<float>, dim3(a.B), dim3(threads), smem, st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_encode_paged(const state::Args& a, bool bf16, const void* rows, int64_t n,
                                int64_t first_entry, cudaStream_t st) {
  if (a.B == 0 || n == 0) return cudaSuccess;
  const int threads = a.c >= 256 ? 256 : ((a.c + 31) / 32) * 32;
  const size_t smem = (size_t)a.c * sizeof(float);
  const dim3 grid((unsigned)n, (unsigned)a.B);
  cudaError_t e = bf16 ? launch(false, k_encode_paged<__nv_bfloat16>, grid, dim3(threads), smem,
                                st, a, rows, n, first_entry)
                       : launch(false, k_encode_paged<float>, grid, dim3(threads), smem, st, a,
                                rows, n, first_entry);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t state_append_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_state_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_state_error, &zero, sizeof(int));
}

}  // namespace csa
