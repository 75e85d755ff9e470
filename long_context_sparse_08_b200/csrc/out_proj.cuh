// Grouped output projection at decode: the layouts, split geometry and per-element
// arithmetic, written once as __host__ __device__ functions for the kernels (out_proj.cu)
// and for a host build the CPU tests compare with the oracle.
//
// 【论文解读】DeepSeek-V4, 一(三)1(4) 分组输出投影 (and 2(2) for HCA): the H head outputs
// o_{t,1..H} [c] are split into g groups of H/g heads; group i (heads i*H/g .. (i+1)*H/g-1,
// concatenated: c*H/g values) is projected to d_g values by its own matrix, and the g*d_g
// concatenation is projected to the output of d values. 三(二) 模型配置: g = 8 / 16,
// d_g = 1024, d = 4096 / 7168 for Flash / Pro.
//
// Layouts (row vectors times matrices, x . W): o bf16 [Q, H*c] (a query's heads in order);
// w_grp bf16 [g, K1 = c*H/g, d_g]; w_out bf16 [g*d_g, d]; out bf16 [Q, d].
// With a few queries (decode) each weight is used Q times: the work streams the weights
// from HBM. A thread owns 8 consecutive output columns (one 16-byte weight load per row) and
// Q x 8 fp32 sums; a warp covers 256 columns of a row; a CTA of 4 warps 1024 columns, over a
// slice of the rows (K split across CTAs; rows in ascending order). Each split writes fp32
// partials; a pass sums stage 1's partials in split order into the fp32 intermediate, and a
// last pass sums stage 2's partials into the bf16 output.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

namespace csa {
namespace proj {

#define CSA_HD __host__ __device__ __forceinline__

constexpr int kColsPerThread = 8;
constexpr int kWarps = 4;
constexpr int kColsPerCta = 32 * kColsPerThread * kWarps;  // 1024

struct Geom {
  int Q, H, c, g, d_g, d;
  int K1;      // c * H / g: rows of a group's matrix
  int S1, S2;  // K splits of stage 1 (over K1) and stage 2 (over g * d_g)
  int ks1, ks2;  // rows per split
};

CSA_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }

constexpr int kMaxRowsPerSplit = 512;  // a split's inputs (<= 16 x 512 fp32) fit 32 KB of smem

// Splits: enough CTAs for about two waves of `sms`, at most kMaxRowsPerSplit rows and at
// least 64 rows per split (where the matrix has them).
CSA_HD Geom make_geom(int Q, int H, int c, int g, int d_g, int d, int sms) {
  Geom G{};
  G.Q = Q; G.H = H; G.c = c; G.g = g; G.d_g = d_g; G.d = d;
  G.K1 = c * (H / g);
  const int K2 = g * d_g;
  const int ctas1 = g * ceil_div(d_g, kColsPerCta), ctas2 = ceil_div(d, kColsPerCta);
  int s1 = ceil_div(2 * sms, ctas1), s2 = ceil_div(2 * sms, ctas2);
  const int max1 = G.K1 / 64 > 0 ? G.K1 / 64 : 1, max2 = K2 / 64 > 0 ? K2 / 64 : 1;
  s1 = s1 > max1 ? max1 : s1;
  s2 = s2 > max2 ? max2 : s2;
  const int min1 = ceil_div(G.K1, kMaxRowsPerSplit), min2 = ceil_div(K2, kMaxRowsPerSplit);
  s1 = s1 < min1 ? min1 : (s1 < 1 ? 1 : s1);
  s2 = s2 < min2 ? min2 : (s2 < 1 ? 1 : s2);
  G.ks1 = ceil_div(G.K1, s1);
  G.ks2 = ceil_div(g * d_g, s2);
  G.S1 = ceil_div(G.K1, G.ks1);
  G.S2 = ceil_div(g * d_g, G.ks2);
  return G;
}

// fp32 elements of the workspace: stage 1's partials, the intermediate, stage 2's partials
CSA_HD size_t part1_elems(const Geom& G) { return (size_t)G.S1 * G.Q * G.g * G.d_g; }
CSA_HD size_t mid_elems(const Geom& G) { return (size_t)G.Q * G.g * G.d_g; }
CSA_HD size_t part2_elems(const Geom& G) { return (size_t)G.S2 * G.Q * G.d; }

// stage 1: element (q, k) of group z's input row = o[q, z*K1 + k]
CSA_HD size_t o_index(const Geom& G, int q, int z, int k) {
  return (size_t)q * G.H * G.c + (size_t)z * G.K1 + k;
}
// weight (k, f) of group z
CSA_HD size_t wgrp_index(const Geom& G, int z, int k, int f) {
  return ((size_t)z * G.K1 + k) * G.d_g + f;
}
// partial of split s, query q, intermediate column z*d_g + f
CSA_HD size_t part1_index(const Geom& G, int s, int q, int col) {
  return ((size_t)s * G.Q + q) * ((size_t)G.g * G.d_g) + col;
}
CSA_HD size_t wout_index(const Geom& G, int k, int f) { return (size_t)k * G.d + f; }
CSA_HD size_t part2_index(const Geom& G, int s, int q, int f) {
  return ((size_t)s * G.Q + q) * (size_t)G.d + f;
}

CSA_HD size_t mid_index(const Geom& G, int q, int k) { return (size_t)q * G.g * G.d_g + k; }

// intermediate value (q, column k) = sum of stage 1's splits in order
CSA_HD float mid_value(const Geom& G, const float* part1, int q, int k) {
  float v = 0.f;
  for (int s = 0; s < G.S1; ++s) v += part1[part1_index(G, s, q, k)];
  return v;
}
// output value (q, f) = sum of stage 2's splits in order
CSA_HD float out_value(const Geom& G, const float* part2, int q, int f) {
  float v = 0.f;
  for (int s = 0; s < G.S2; ++s) v += part2[part2_index(G, s, q, f)];
  return v;
}

// 8 bf16 weights (one 16-byte load) -> floats
CSA_HD void widen8(const uint4& w, float (&x)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = u[i] << 16, hi = u[i] & 0xffff0000u;
    float a, b;
    memcpy(&a, &lo, 4);
    memcpy(&b, &hi, 4);
    x[2 * i] = a;
    x[2 * i + 1] = b;
  }
}

#undef CSA_HD

}  // namespace proj

struct OutProjArgs {
  proj::Geom G;
  const __nv_bfloat16 *o, *w_grp, *w_out;
  __nv_bfloat16* out;
  float *part1, *mid, *part2;  // workspace
};

}  // namespace csa
