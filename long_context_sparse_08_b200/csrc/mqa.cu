// Stage 4: shared-KV MQA over compressed entries plus the sliding window, with sink.
//
// 【论文解读】DeepSeek-V4:
//   一(三)1(3) Shared Key-Value MQA -- every selected entry is both key and value for all
//     n_h query heads; 一(三)2(2) HCA -- the same over every visible entry;
//   一(三)3(1) RMSNorm of each query head; 3(2) RoPE(t) on the last r dims of q and
//     RoPE(-t) on the last r dims of each head's output; 3(3) the n_win most recent
//     uncompressed tokens are attended together with the compressed entries;
//   3(4) the sink: exp(z'_h) is added to the softmax denominator.
//
// This version runs on CUDA cores: one CTA per (query, group of up to 16 heads); the KV
// rows of the query (selected or all visible entries, then the window) stream through
// shared memory in chunks of 32 rows with an online (running-max) softmax; each thread
// owns two output dims of every head of the group.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;   // KV rows per chunk
constexpr int kMaxHpb = 16; // heads per CTA

struct RowRef {
  const void* ptr;  // row base, or nullptr when the slot holds no valid row
};

template <typename T>
__global__ void __launch_bounds__(kThreads) k_mqa_cc(MqaArgs a) {
  extern __shared__ float sm[];
  const int c = a.c;
  const int hpb = a.H < kMaxHpb ? a.H : kMaxHpb;
  float* qs = sm;                       // [hpb, c]
  float* rows = qs + kMaxHpb * c;       // [kRows, c]
  float* z = rows + kRows * c;          // [hpb, kRows]
  float* alpha = z + kMaxHpb * kRows;   // [hpb]
  float* mrun = alpha + kMaxHpb;        // [hpb]
  float* lrun = mrun + kMaxHpb;         // [hpb]
  int* valid = reinterpret_cast<int*>(lrun + kMaxHpb);  // [kRows]
  __shared__ float red[32];

  const int bt = blockIdx.y;
  const int b = bt / a.T;
  const int h0 = blockIdx.x * hpb;
  const int64_t t = a.q_pos[bt];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const T* q = static_cast<const T*>(a.q) + ((size_t)bt * a.H + h0) * c;
  const T* kvb = static_cast<const T*>(a.kv) + (size_t)b * a.n_cap * c;
  const T* winb = static_cast<const T*>(a.win) + (size_t)b * a.l_raw * c;
  const int64_t pos0 = a.win_pos0[b];
  const int64_t n_vis = t < 0 ? 0 : (t / a.m < a.n_cap ? t / a.m : a.n_cap);
  const int64_t n_sel = a.k > 0 ? a.k : n_vis;
  const int64_t lo = (t - a.n_win + 1) > 0 ? (t - a.n_win + 1) : 0;
  const int64_t n_w = a.n_win > 0 && t >= 0 ? t - lo + 1 : 0;
  const int64_t L = n_sel + n_w;
  const int32_t* idx = a.idx ? a.idx + (size_t)bt * a.k : nullptr;
  const T* g = static_cast<const T*>(a.q_rms_w);

  // ---- query prep: RMSNorm per head, then RoPE(t) on the last r dims ----
  for (int e = tid; e < hpb * c; e += blockDim.x) qs[e] = to_f32(q[e]);
  __syncthreads();
  for (int h = wid; h < hpb; h += blockDim.x / 32) {
    float ss = 0.f;
    for (int j = lane; j < c; j += 32) ss = fmaf(qs[h * c + j], qs[h * c + j], ss);
    ss = warp_sum(ss);
    const float rstd = rsqrtf(ss / (float)c + a.eps);
    for (int j = lane; j < c; j += 32) qs[h * c + j] *= rstd * (g ? to_f32(g[j]) : 1.f);
  }
  __syncthreads();
  const int r = a.rope_dims, r0 = c - r;
  for (int e = tid; e < hpb * (r / 2); e += blockDim.x) {
    const int h = e / (r / 2), p = e % (r / 2);
    float cs, sn;
    rope_cos_sin((double)t, p, r, (double)a.rope_base, &cs, &sn);
    float* x = qs + h * c + r0 + 2 * p;
    const float x0 = x[0], x1 = x[1];
    x[0] = x0 * cs - x1 * sn;
    x[1] = x0 * sn + x1 * cs;
  }
  if (tid < hpb) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.f;
  }
  // each thread owns output dims (2*tid, 2*tid+1) of every head in the group
  const bool owns = 2 * tid < c;
  float o[kMaxHpb][2];
#pragma unroll
  for (int h = 0; h < kMaxHpb; ++h) o[h][0] = o[h][1] = 0.f;
  __syncthreads();

  for (int64_t base = 0; base < L; base += kRows) {
    // ---- stage the chunk's rows (fp32) ----
    if (tid < kRows) {
      const int64_t j = base + tid;
      const T* src = nullptr;
      if (j < n_sel) {
        const int64_t e = idx ? (int64_t)idx[j] : j;
        if (e >= 0 && e < a.n_cap) src = kvb + (size_t)e * c;
      } else if (j < L) {
        const int64_t rr = lo + (j - n_sel) - pos0;
        if (rr >= 0 && rr < a.l_raw) src = winb + (size_t)rr * c;
      }
      valid[tid] = src != nullptr;
      reinterpret_cast<const T**>(z)[tid] = src;  // z doubles as the pointer table here
    }
    __syncthreads();
    const T* const* srcs = reinterpret_cast<const T* const*>(z);
    for (int e = tid; e < kRows * c; e += blockDim.x) {
      const int rr = e / c, j = e % c;
      const T* s = srcs[rr];
      rows[e] = s ? to_f32(s[j]) : 0.f;
    }
    __syncthreads();
    // ---- logits: warp w handles heads w, w+8, ...; lane-split dot over c ----
    for (int h = wid; h < hpb; h += blockDim.x / 32) {
      for (int rr = 0; rr < kRows; ++rr) {
        float d = 0.f;
        for (int j = lane; j < c; j += 32) d = fmaf(qs[h * c + j], rows[rr * c + j], d);
        d = warp_sum(d);
        if (lane == 0) z[h * kRows + rr] = valid[rr] ? d * a.scale : -INFINITY;
      }
    }
    __syncthreads();
    // ---- online softmax bookkeeping per head ----
    if (tid < hpb) {
      const int h = tid;
      float cm = -INFINITY;
      for (int rr = 0; rr < kRows; ++rr) cm = fmaxf(cm, z[h * kRows + rr]);
      const float mnew = fmaxf(mrun[h], cm);
      float al = 1.f, sum = 0.f;
      if (mnew != -INFINITY) {
        al = mrun[h] == -INFINITY ? 0.f : expf(mrun[h] - mnew);
        for (int rr = 0; rr < kRows; ++rr) {
          const float p = z[h * kRows + rr] == -INFINITY ? 0.f : expf(z[h * kRows + rr] - mnew);
          z[h * kRows + rr] = p;
          sum += p;
        }
      } else {
        for (int rr = 0; rr < kRows; ++rr) z[h * kRows + rr] = 0.f;
      }
      alpha[h] = al;
      mrun[h] = mnew;
      lrun[h] = lrun[h] * al + sum;
    }
    __syncthreads();
    // ---- o = o * alpha + P . rows ----
    if (owns) {
#pragma unroll
      for (int h = 0; h < kMaxHpb; ++h)
        if (h < hpb) {
          o[h][0] *= alpha[h];
          o[h][1] *= alpha[h];
        }
      for (int rr = 0; rr < kRows; ++rr) {
        const float v0 = rows[rr * c + 2 * tid], v1 = rows[rr * c + 2 * tid + 1];
#pragma unroll
        for (int h = 0; h < kMaxHpb; ++h)
          if (h < hpb) {
            const float p = z[h * kRows + rr];
            o[h][0] = fmaf(p, v0, o[h][0]);
            o[h][1] = fmaf(p, v1, o[h][1]);
          }
      }
    }
    __syncthreads();
  }

  // ---- finalise: divide by (l + e^{sink - m}) and rotate by -t ----
  if (owns) {
    T* out = static_cast<T*>(a.out) + ((size_t)bt * a.H + h0) * c;
    const int j0 = 2 * tid;
    float cs = 1.f, sn = 0.f;
    if (j0 >= r0) rope_cos_sin(-(double)t, (j0 - r0) >> 1, r, (double)a.rope_base, &cs, &sn);
#pragma unroll
    for (int h = 0; h < kMaxHpb; ++h)
      if (h < hpb) {
        const float zs = a.sink ? a.sink[h0 + h] : -INFINITY;
        const float m = mrun[h];
        float y0 = 0.f, y1 = 0.f;
        if (lrun[h] > 0.f) {
          const float M = fmaxf(m, zs);
          const float f = expf(m - M);
          const float den = lrun[h] * f + (zs == -INFINITY ? 0.f : expf(zs - M));
          y0 = o[h][0] * f / den;
          y1 = o[h][1] * f / den;
        }
        const float u0 = y0 * cs - y1 * sn, u1 = y0 * sn + y1 * cs;
        out[(size_t)h * c + j0] = from_f32<T>(u0);
        out[(size_t)h * c + j0 + 1] = from_f32<T>(u1);
      }
  }
  (void)red;
}

}  // namespace

size_t mqa_workspace_bytes(const MqaArgs& a) {
  // sized for the tensor-core path whenever its shape constraints hold (bf16 or not)
  return mqa_tc_supported(a, true) ? mqa_tc_workspace_bytes(a) : 0;
}

cudaError_t launch_mqa(const MqaArgs& a, bool bf16, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (a.B == 0 || a.T == 0 || a.H == 0) return cudaSuccess;
  if (mqa_tc_supported(a, bf16)) return launch_mqa_tc(a, ws, ws_bytes, st);
  const int hpb = a.H < kMaxHpb ? a.H : kMaxHpb;
  dim3 grid(a.H / hpb, a.B * a.T);
  const size_t smem = ((size_t)kMaxHpb * a.c + (size_t)kRows * a.c + kMaxHpb * kRows +
                       3 * kMaxHpb + kRows) * sizeof(float);
  cudaError_t e;
  if (bf16) {
    e = cudaFuncSetAttribute(k_mqa_cc<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    launch(false, k_mqa_cc<__nv_bfloat16>, dim3(grid), dim3(kThreads), smem, st, a);
  } else {
    e = cudaFuncSetAttribute(k_mqa_cc<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    launch(false, k_mqa_cc<float>, dim3(grid), dim3(kThreads), smem, st, a);
  }
  return cudaGetLastError();
}

}  // namespace csa
