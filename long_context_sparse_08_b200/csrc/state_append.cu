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

enum { kErrBase = 300 };  // stored code = kErrBase - status (301 position, 302 page slot, 303 page id)

template <typename T>
__global__ void __launch_bounds__(256) k_state_append(state::Args a) {
  extern __shared__ float row[];  // [c]
  __shared__ float red[32];
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
  T* out = static_cast<T*>(a.pages) + off;
  if (!a.finalize) {
    for (int j = threadIdx.x; j < a.c; j += blockDim.x) state::st(out, j, row[j]);
    return;
  }
  const float tot = block_sum(ss, red);  // also orders the row[] writes before the reads
  const float rstd = rsqrtf(tot / (float)a.c + a.eps);
  for (int j = threadIdx.x; j < a.c; j += blockDim.x)
    state::st(out, j, state::final_channel<T>(a, row, rstd, i, j));
}

}  // namespace

cudaError_t launch_state_append(const state::Args& a, bool bf16, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  const int threads = a.c >= 256 ? 256 : ((a.c + 31) / 32) * 32;
  const size_t smem = (size_t)a.c * sizeof(float);
  cudaError_t e = bf16 ? launch(false, k_state_append<__nv_bfloat16>, dim3(a.B), dim3(threads),
                                smem, st, a)
                       : launch(false, k_state_append<float>, dim3(a.B), dim3(threads), smem, st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t state_append_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_state_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_state_error, &zero, sizeof(int));
}

}  // namespace csa
