// Grouped output projection at decode (【论文解读】DeepSeek-V4, 一(三)1(4) 分组输出投影): the
// kernels. Layouts, split geometry and index arithmetic live in out_proj.cuh.
//
// HBM-bound weight streaming on CUDA cores: with Q <= 16 queries a weight byte carries
// 2 Q / 2 flops, far below the tensor cores' ridge, so the kernels size for coalesced 16-byte
// loads and bytes in flight: a thread owns 8 output columns and Q x 8 fp32 sums, reads one
// 16-byte row segment per step (8 rows in flight), and takes its inputs from shared memory
// (every lane of a warp reads the same value: a broadcast). Splits of the rows go to
// separate CTAs, about two waves of the SMs; the partial sums are added in a fixed order, so
// results do not depend on the schedule.
#include "common.cuh"
#include "host_util.cuh"
#include "internal.h"
#include "out_proj.cuh"

namespace csa {

namespace {

using proj::Geom;

// One split of rows [k0, k1) of one matrix: stage 1 (kStage2 = false) for group z = blockIdx.x,
// inputs o; stage 2 for column block blockIdx.x, inputs the intermediate.
template <int QM, bool kStage2>
__global__ void __launch_bounds__(128) k_out_proj_split(OutProjArgs a) {
  extern __shared__ float xs[];  // [QM][ks] inputs of this split
  const Geom& G = a.G;
  const int s = blockIdx.y;
  const int K = kStage2 ? G.g * G.d_g : G.K1;
  const int ks = kStage2 ? G.ks2 : G.ks1;
  const int F = kStage2 ? G.d : G.d_g;
  const int z = kStage2 ? 0 : (int)blockIdx.x / proj::ceil_div(G.d_g, proj::kColsPerCta);
  const int cb = kStage2 ? (int)blockIdx.x : (int)blockIdx.x % proj::ceil_div(G.d_g, proj::kColsPerCta);
  const int k0 = s * ks, k1 = min(K, k0 + ks), nk = k1 - k0;
  for (int i = threadIdx.x; i < G.Q * nk; i += blockDim.x) {
    const int q = i / nk, kk = i - q * nk;
    xs[q * ks + kk] =
        kStage2 ? a.mid[proj::mid_index(G, q, k0 + kk)]
                : __bfloat162float(a.o[proj::o_index(G, q, z, k0 + kk)]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f0 = cb * proj::kColsPerCta + warp * 256 + lane * proj::kColsPerThread;
  if (f0 >= F) return;
  float acc[QM][8];
#pragma unroll
  for (int q = 0; q < QM; ++q)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[q][i] = 0.f;
  const __nv_bfloat16* W = kStage2 ? a.w_out : a.w_grp;
  auto widx = [&](int k) {
    return kStage2 ? proj::wout_index(G, k, f0) : proj::wgrp_index(G, z, k, f0);
  };
  constexpr int kU = 8;  // rows in flight per thread
  int k = k0;
  for (; k + kU <= k1; k += kU) {
    uint4 w[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) w[u] = __ldg(reinterpret_cast<const uint4*>(W + widx(k + u)));
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      float wv[8];
      proj::widen8(w[u], wv);
#pragma unroll
      for (int q = 0; q < QM; ++q) {
        if (q < G.Q) {
          const float x = xs[q * ks + (k + u - k0)];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[q][i] = fmaf(x, wv[i], acc[q][i]);
        }
      }
    }
  }
  for (; k < k1; ++k) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(W + widx(k)));
    float wv[8];
    proj::widen8(w, wv);
#pragma unroll
    for (int q = 0; q < QM; ++q) {
      if (q < G.Q) {
        const float x = xs[q * ks + (k - k0)];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[q][i] = fmaf(x, wv[i], acc[q][i]);
      }
    }
  }
  const int col = kStage2 ? f0 : z * G.d_g + f0;
#pragma unroll
  for (int q = 0; q < QM; ++q) {
    if (q < G.Q) {
      float* dst = kStage2 ? a.part2 + proj::part2_index(G, s, q, col)
                           : a.part1 + proj::part1_index(G, s, q, col);
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[q][4], acc[q][5], acc[q][6], acc[q][7]);
    }
  }
}

// Sum of the splits in order: stage 1 into the fp32 intermediate, stage 2 into bf16 out.
template <bool kStage2>
__global__ void __launch_bounds__(256) k_out_proj_reduce(OutProjArgs a) {
  const Geom& G = a.G;
  const int n = kStage2 ? G.d : G.g * G.d_g;
  const int64_t total = (int64_t)G.Q * n;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int q = (int)(i / n), f = (int)(i - (int64_t)q * n);
    if (kStage2)
      a.out[(size_t)q * G.d + f] = __float2bfloat16_rn(proj::out_value(G, a.part2, q, f));
    else
      a.mid[proj::mid_index(G, q, f)] = proj::mid_value(G, a.part1, q, f);
  }
}

template <int QM>
cudaError_t launch_splits(const OutProjArgs& a, cudaStream_t st) {
  const Geom& G = a.G;
  const size_t smem1 = (size_t)QM * G.ks1 * sizeof(float);
  const size_t smem2 = (size_t)QM * G.ks2 * sizeof(float);
  const dim3 grid1(G.g * proj::ceil_div(G.d_g, proj::kColsPerCta), G.S1);
  const dim3 grid2(proj::ceil_div(G.d, proj::kColsPerCta), G.S2);
  const int red_blocks = 2 * device_sm_count();
  cudaError_t e = launch(false, k_out_proj_split<QM, false>, grid1, dim3(128), smem1, st, a);
  if (e == cudaSuccess)
    e = launch(false, k_out_proj_reduce<false>, dim3(red_blocks), dim3(256), 0, st, a);
  if (e == cudaSuccess)
    e = launch(false, k_out_proj_split<QM, true>, grid2, dim3(128), smem2, st, a);
  if (e == cudaSuccess)
    e = launch(false, k_out_proj_reduce<true>, dim3(red_blocks), dim3(256), 0, st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

proj::Geom out_proj_geom(int Q, int H, int c, int g, int d_g, int d) {
  return proj::make_geom(Q, H, c, g, d_g, d, device_sm_count());
}

size_t out_proj_workspace_bytes(const proj::Geom& G) {
  return (proj::part1_elems(G) + proj::mid_elems(G) + proj::part2_elems(G)) * sizeof(float) + 3 * 256;
}

cudaError_t launch_out_proj(OutProjArgs a, void* ws, cudaStream_t st) {
  const Geom& G = a.G;
  auto align = [](size_t x) { return (x + 255) / 256 * 256; };
  char* p = static_cast<char*>(ws);
  a.part1 = reinterpret_cast<float*>(p);
  p += align(proj::part1_elems(G) * sizeof(float));
  a.mid = reinterpret_cast<float*>(p);
  p += align(proj::mid_elems(G) * sizeof(float));
  a.part2 = reinterpret_cast<float*>(p);
  if (G.Q <= 4) return launch_splits<4>(a, st);
  if (G.Q <= 8) return launch_splits<8>(a, st);
  return launch_splits<16>(a, st);
}

}  // namespace csa
