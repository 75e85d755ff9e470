// q_hat = RoPE_t(RMSNorm(q) * q_rms_w) rows in bf16 for the tensor-core attention, as a
// side job of the top-k kernels that precede it (【论文解读】DeepSeek-V4 一(三)3(1), 3(2)).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace csa {

// One head's q_hat row from its raw bf16 row (lane holds dims 8*lane.. and 256 + 8*lane..).
__device__ __forceinline__ void qhat_head(const QhatJob& j, const uint4 (&raw)[2], uint4* dst,
                                          const float* cs, const float* sn) {
  constexpr int kC = 512;
  const int lane = threadIdx.x & 31;
  const int r0 = kC - j.r;
  float ss = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t w4[4] = {raw[half].x, raw[half].y, raw[half].z, raw[half].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(w4[k] << 16), hi = __uint_as_float(w4[k] & 0xffff0000u);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
  }
  ss = warp_sum(ss);
  const float rstd = rsqrtf(ss / (float)kC + j.eps);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int d0 = 8 * (lane + 32 * half);
    const uint32_t w4[4] = {raw[half].x, raw[half].y, raw[half].z, raw[half].w};
    float y[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float x = (k & 1) ? __uint_as_float(w4[k >> 1] & 0xffff0000u)
                              : __uint_as_float(w4[k >> 1] << 16);
      const float wgt =
          j.q_rms_w ? __bfloat162float(static_cast<const __nv_bfloat16*>(j.q_rms_w)[d0 + k]) : 1.f;
      y[k] = x * rstd * wgt;
    }
    if (d0 >= r0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int p = (d0 + 2 * k - r0) >> 1;
        const float c = cs[p], s = sn[p], u = y[2 * k], v = y[2 * k + 1];
        y[2 * k] = u * c - v * s;
        y[2 * k + 1] = u * s + v * c;
      }
    }
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      ow[k] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * k])) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * k + 1])) << 16);
    dst[lane + 32 * half] = o;
  }
}

// The side job: q_hat rows of query q for heads [h0, h1), one warp per head, lane = 16 of
// the 512 dims; a warp reads two heads' rows before working on either, so each round trip
// to memory serves two heads. Reads only caller inputs, so it runs before the dependency
// wait.
__device__ inline void qhat_rows(const QhatJob& j, int q, double t, int h0, int h1, float* cs,
                                 float* sn) {
  constexpr int kC = 512;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nwarps = blockDim.x >> 5;
  for (int p = tid; p < j.r / 2; p += blockDim.x) rope_angle_cs(t, j.inv_freq[p], &cs[p], &sn[p]);
  __syncthreads();
  for (int h = h0 + wid; h < h1; h += 2 * nwarps) {
    const int h2 = h + nwarps;
    const uint4* src = reinterpret_cast<const uint4*>(j.q) + ((size_t)q * j.H + h) * (kC / 8);
    const uint4* src2 = reinterpret_cast<const uint4*>(j.q) + ((size_t)q * j.H + h2) * (kC / 8);
    uint4 ra[2], rb[2];
    ra[0] = src[lane];
    ra[1] = src[lane + 32];
    if (h2 < h1) {
      rb[0] = src2[lane];
      rb[1] = src2[lane + 32];
    }
    qhat_head(j, ra, reinterpret_cast<uint4*>(j.qhat) + ((size_t)q * j.H + h) * (kC / 8), cs, sn);
    if (h2 < h1)
      qhat_head(j, rb, reinterpret_cast<uint4*>(j.qhat) + ((size_t)q * j.H + h2) * (kC / 8), cs,
                sn);
  }
}

}  // namespace csa
