// Stage 2: lightning-indexer scores on CUDA cores.
//
// 【论文解读】DeepSeek-V4, 一(三)1(2) Lightning Indexer 稀疏选择:
//   I[t,s] = sum_h w[t,h] * ReLU(q^I[t,h] . K^IComp[s]),  for s < floor(t/m).
// The keys are read in the stored format (fp32, bf16, or e4m3 with a row scale) and
// decoded exactly in registers; every product is exact in fp32 and the sums are fp32.
// (MXFP4 keys go through the tensor-core kernel of indexer_mxf4.cu.) For e4m3 keys the row scale is applied after the dot
// product (ReLU(s*x) = s*ReLU(x) for s >= 0), so no product is rounded.
//
// One thread per key, 128 keys per CTA, one (request, query) per grid row; the query's
// decoded heads [H_I, d_I] sit in shared memory and are read as broadcasts.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kKeysPerCta = 128;
constexpr int kHeadGroup = 16;
constexpr int kChunk = 32;

// Decode 32 consecutive key elements [d0, d0+32) of key row `s` into fp32.
template <int KDT>
__device__ __forceinline__ void load_key_chunk(const IndexArgs& a, int b, int64_t s, int d0,
                                               float* v) {
  const int d = a.d_idx;
  const size_t row = (size_t)b * a.n_cap + s;
  if (KDT == CSA_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(a.KI) +
                                                      row * d + d0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 x = p[q];
      v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
    }
  } else if (KDT == CSA_BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(
        static_cast<const __nv_bfloat16*>(a.KI) + row * d + d0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 x = p[q];
      const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[8 * q + 2 * k] = __uint_as_float(w4[k] << 16);
        v[8 * q + 2 * k + 1] = __uint_as_float(w4[k] & 0xffff0000u);
      }
    }
  } else if (KDT == CSA_FP8_E4M3_ROWSCALE) {  // raw code values; the row scale comes later
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.KI) +
                                                    row * d + d0);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 x = p[q];
      const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int by = 0; by < 4; ++by)
          v[16 * q + 4 * k + by] = e4m3_to_f32((w4[k] >> (8 * by)) & 0xff);
    }
  }
}

template <int KDT>
__global__ void __launch_bounds__(kKeysPerCta) k_index_scores_cc(IndexArgs a) {
  extern __shared__ float qs[];  // [H_I * d_I] decoded queries, then [H_I] weights
  const int bt = blockIdx.y;
  const int b = bt / a.T;
  const int64_t t = a.q_pos[bt];
  const int64_t n_vis = t < 0 ? 0 : (t / a.m < a.n_cap ? t / a.m : a.n_cap);
  const int64_t s0 = (int64_t)blockIdx.x * kKeysPerCta;
  if (s0 >= n_vis) return;
  const int H = a.n_idx_heads, d = a.d_idx;
  float* ws = qs + H * d;
  // decode this query's indexer heads into shared memory
  for (int e = threadIdx.x; e < H * d; e += blockDim.x) {
    float v;
    const size_t off = (size_t)bt * H * d + e;
    if (KDT == CSA_F32) {
      v = static_cast<const float*>(a.qI)[off];
    } else {
      v = to_f32(static_cast<const __nv_bfloat16*>(a.qI)[off]);
    }
    qs[e] = v;
  }
  for (int h = threadIdx.x; h < H; h += blockDim.x) ws[h] = a.w[(size_t)bt * H + h];
  __syncthreads();

  const int64_t s = s0 + threadIdx.x;
  if (s >= n_vis) return;
  float score = 0.f;
  const int hg_n = H < kHeadGroup ? H : kHeadGroup;
  for (int hg = 0; hg < H; hg += hg_n) {
    float acc[kHeadGroup];
#pragma unroll
    for (int h = 0; h < kHeadGroup; ++h) acc[h] = 0.f;
    for (int d0 = 0; d0 < d; d0 += kChunk) {
      float kv[kChunk];
      load_key_chunk<KDT>(a, b, s, d0, kv);
#pragma unroll
      for (int h = 0; h < kHeadGroup; ++h) {
        if (h < hg_n) {
          const float* qh = qs + (hg + h) * d + d0;
#pragma unroll
          for (int j = 0; j < kChunk; ++j) acc[h] = fmaf(kv[j], qh[j], acc[h]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kHeadGroup; ++h)
      if (h < hg_n) score = fmaf(ws[hg + h], fmaxf(acc[h], 0.f), score);
  }
  if (KDT == CSA_FP8_E4M3_ROWSCALE)
    score *= static_cast<const float*>(a.KI_scale)[(size_t)b * a.n_cap + s];
  a.scores[(size_t)bt * a.n_cap + s] = score;
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, cudaStream_t st, bool* hist_done) {
  if (hist_done) *hist_done = false;
  if (a.B == 0 || a.T == 0 || a.n_cap == 0) return cudaSuccess;
  if (index_mxf4_tc_supported(a)) {  // MXFP4 keys (contiguous or paged; fp32 or bf16 scores)
    if (hist_done) *hist_done = a.hist != nullptr;
    return launch_index_mxf4_tc(a, st);
  }
  if (a.scores16 != nullptr || a.page_table != nullptr) {
    // BF16 index scores or paged keys otherwise: the FP8 / bf16 tensor-core kernel only
    if (!index_bf16_tc_supported(a)) return cudaErrorNotSupported;
    if (hist_done) *hist_done = a.hist != nullptr;
    return launch_index_bf16_tc(a, st);
  }
  if (index_bf16_tc_supported(a)) {
    if (hist_done) *hist_done = a.hist != nullptr;
    return launch_index_bf16_tc(a, st);
  }
  dim3 grid((unsigned)((a.n_cap + kKeysPerCta - 1) / kKeysPerCta), a.B * a.T);
  const size_t smem = ((size_t)a.n_idx_heads * a.d_idx + a.n_idx_heads) * sizeof(float);
  timing_before(st);
  switch (a.kdt) {
    case CSA_F32:
      launch(false, k_index_scores_cc<CSA_F32>, dim3(grid), dim3(kKeysPerCta), smem, st, a);
      break;
    case CSA_BF16:
      launch(false, k_index_scores_cc<CSA_BF16>, dim3(grid), dim3(kKeysPerCta), smem, st, a);
      break;
    default:
      launch(false, k_index_scores_cc<CSA_FP8_E4M3_ROWSCALE>, dim3(grid), dim3(kKeysPerCta),
             smem, st, a);
      break;
  }
  timing_after(st);
  return cudaGetLastError();
}

}  // namespace csa
