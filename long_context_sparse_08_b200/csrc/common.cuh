// Device helpers shared by the kernels of libcsa (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

constexpr int kMaxTopk = 2048;

// ---------------------------------------------------------------------------
// element access
// ---------------------------------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// OCP e4m3 ("fn") code -> float, exact: normal (8+f) * 2^(e-10), subnormal f * 2^-9.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xF, f = code & 7;
  float mag = (e == 0) ? (float)f * 0.001953125f
                       : __uint_as_float(((e + 120u) << 23) | (f << 20));
  if (e == 15 && f == 7) mag = __uint_as_float(0x7fc00000u);
  return (code & 0x80) ? -mag : mag;
}

// OCP e2m1 nibble -> float (exact): magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
__device__ __forceinline__ float e2m1_to_f32(uint32_t nib) {
  const uint32_t e = (nib >> 1) & 3, f = nib & 1;
  float mag = (e == 0) ? 0.5f * (float)f : __uint_as_float(((e + 126u) << 23) | (f << 22));
  return (nib & 8) ? -mag : mag;
}

// e8m0 scale byte -> 2^(b-127) (255 -> NaN); 0 -> 2^-127 (a subnormal float).
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
  if (b == 255) return __uint_as_float(0x7fc00000u);
  if (b == 0) return __uint_as_float(0x00400000u);
  return __uint_as_float(b << 23);
}

// An index score of either storage type, widened to fp32 (bf16 -> fp32 is exact).
__device__ __forceinline__ float ld_score(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_score(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

// Order-preserving map of a float to uint32 (larger float -> larger key). -0 maps like +0.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched with the programmatic stream
// serialisation attribute may start while its predecessor in the stream still runs;
// pdl_wait() returns once every prerequisite grid has completed and its writes are
// visible, pdl_trigger() lets the next such kernel start. Both do nothing in a kernel
// launched the ordinary way.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum; `red` is shared scratch of >= 32 floats. All threads get the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.f;
  if (wid == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

// ---------------------------------------------------------------------------
// RoPE angles. Pair p of the last r dims turns by pos * base^(-2p/r). The angle reaches
// ~1e6 rad at 1M positions, so it is formed in double and reduced modulo 2*pi with a
// two-part 2*pi (Cody-Waite); the reduced angle (|a| <= pi) then goes through fp32
// sincosf. Error ~1e-10 rad before the fp32 evaluation, which adds ~1 ulp.
// ---------------------------------------------------------------------------
__host__ __device__ inline double rope_inv_freq(int p, int r, double base) {
  return exp2(-2.0 * (double)p / (double)r * log2(base));
}
__device__ __forceinline__ void rope_angle_cs(double pos, double inv_freq, float* cs, float* sn) {
  const double x = pos * inv_freq;
  const double kTwoPiHi = 6.283185307179586232;     // nearest double to 2*pi
  const double kTwoPiLo = 2.4492935982947064e-16;   // 2*pi - kTwoPiHi
  const double k = rint(x * 0.15915494309189535);   // x / (2*pi)
  double red = fma(-k, kTwoPiHi, x);
  red = fma(-k, kTwoPiLo, red);
  sincosf((float)red, sn, cs);
}
__device__ __forceinline__ void rope_cos_sin(double pos, int p, int r, double base, float* cs,
                                             float* sn) {
  rope_angle_cs(pos, rope_inv_freq(p, r, base), cs, sn);
}

}  // namespace csa
