// Grouped output projection for prefill (many queries) on tensor cores.
//
// 【论文解读】DeepSeek-V4, 一(三)1(4) 分组输出投影: o' = [o_group_i . W_i]_i (g groups), then
// out = o' . W_out. With Q >= 128 queries this is a dense contraction (2 Q flops per weight
// value): two bf16 GEMMs with fp32 accumulation in TMEM,
//   stage 1 (batched over the g groups): mid[:, i*d_g + n] = o[:, i*K1 + k] . W_i[k, n]
//   stage 2:                             out[:, n]        = mid[:, k] . W_out[k, n]
// and the intermediate stored once in bf16.
//
// C[M x N] = A[M x K] . B[K x N]: A (activations) is K-major (a row's K values contiguous),
// B (weights, x . W layout: a row of N values per k) is MN-major. Per CTA tile of 128 rows x
// 256 columns and per 64-wide K step: one 16 KB A box (128 rows x 128 B, 128B-swizzled) and
// four 8 KB B boxes (64 k-rows x 64 n each, 128B-swizzled), four tcgen05 kind::f16 MMAs
// (M = 128, N = 256, K = 16; B read MN-major: 64-element chunks 8 KB apart, 8-row groups
// 1 KB apart, a K step 2 KB).
//
// Persistent: one CTA per SM, 6 warps:
//   warp 0     TMA producer (4-stage ring of 48 KB);
//   warp 1     TMEM (2 accumulators x 256 columns) and the MMA issuer (one lane);
//   warps 2-5  epilogue: TMEM lane quadrant warp % 4 -> 64 columns at a time -> bf16 store.
// Tiles run over (batch, column tile, row tile), row tiles innermost so consecutive CTAs
// share a weight tile in L2. Every wait is bounded and records an error code on expiry.
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "host_util.cuh"
#include "internal.h"
#include "out_proj.cuh"
#include "tc.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;      // 16 KB
constexpr int kBChunkBytes = kBK * 64 * 2;  // 8 KB: 64 k-rows x 64 n
constexpr int kBBytes = 4 * kBChunkBytes;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

enum { kErrFull = 401, kErrEmpty = 402, kErrTFull = 403, kErrTEmpty = 404, kErrDone = 405 };

struct GemmParams {
  int M, N, K;     // per batch
  int batches;
  int a_zx;        // A column offset per batch (elements)
  int b_zy;        // B row offset per batch
  int c_zx;        // C column offset per batch
  int ldc;         // C row stride (elements)
  __nv_bfloat16* C;
};

struct SmemG {
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], done;
  uint32_t tmem_slot;
};

__global__ void __launch_bounds__(kThreads, 1)
    k_out_proj_tc(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  SmemG& S = *reinterpret_cast<SmemG*>(base + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = (p.M + kBM - 1) / kBM, NT = (p.N + kBN - 1) / kBN, KB = (p.K + kBK - 1) / kBK;
  const int tiles = p.batches * NT * MT;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&S.full[i], 1);
        mbar_init(&S.empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&S.tfull[i], 1);
        mbar_init(&S.tempty[i], 4);
      }
      mbar_init(&S.done, 1);
      fence_barrier_init();
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
    }
  } else if (warp == 1) {
    tmem_alloc(&S.tmem_slot, kTmemCols);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int mt = t % MT, nt = (t / MT) % NT, z = t / (MT * NT);
        for (int kb = 0; kb < KB && ok; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&S.empty[s], ((uint32_t)(it / kStages) & 1) ^ 1, kErrEmpty);
          if (!ok) break;
          uint8_t* st = base + s * kStageBytes;
          mbar_arrive_expect_tx(&S.full[s], kStageBytes);
          tma_load_2d(st, &tm_a, z * p.a_zx + kb * kBK, mt * kBM, &S.full[s]);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tma_load_2d(st + kABytes + j * kBChunkBytes, &tm_b, nt * kBN + 64 * j,
                        z * p.b_zy + kb * kBK, &S.full[s]);
        }
      }
      // drain: no copy into this CTA's shared memory may still be in flight at exit
      for (int j = (it > kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait(&S.full[j % kStages], (uint32_t)((j / kStages) & 1), kErrFull);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(1, kBM, kBN) | (1u << 16);  // B MN-major
      const uint32_t sb = smem_u32(base);
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
        const int acc = lt & 1;
        ok = mbar_wait(&S.tempty[acc], ((uint32_t)(lt >> 1) & 1) ^ 1, kErrTEmpty);
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < KB && ok; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&S.full[s], (uint32_t)(it / kStages) & 1, kErrFull);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_s = sb + s * kStageBytes, b_s = a_s + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(a_s + kk * 32, 16, 1024, kLayoutSw128);
            const uint64_t bd = smem_desc(b_s + kk * 2048, kBChunkBytes, 1024, kLayoutSw128);
            mma_f16(tmem + (uint32_t)(kBN * acc), ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&S.empty[s]);
        }
        mma_commit(&S.tfull[acc]);
      }
      mma_commit(&S.done);  // every MMA this thread issued has completed once it fires
      mbar_wait(&S.done, 0, kErrDone);
    }
    __syncwarp();
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
      const int mt = t % MT, nt = (t / MT) % NT, z = t / (MT * NT);
      const int acc = lt & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&S.tfull[acc], (uint32_t)(lt >> 1) & 1, kErrTFull));
      if (!ok) break;
      tc_fence_after();
      const int row = mt * kBM + 32 * quad + lane;
      __nv_bfloat16* crow = p.C + (size_t)row * p.ldc + z * p.c_zx;
#pragma unroll 1
      for (int ch = 0; ch < kBN / 64; ++ch) {
        uint32_t v[64];
        tmem_ld_32x32b_x64(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(kBN * acc + 64 * ch), v);
        tmem_ld_wait();
        const int n0 = nt * kBN + 64 * ch;
        if (row < p.M) {
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8) {
            const int n = n0 + 8 * q8;
            if (n < p.N) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                    __uint_as_float(v[8 * q8 + 2 * i]), __uint_as_float(v[8 * q8 + 2 * i + 1]));
                w[i] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(crow + n) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.tempty[acc]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// bf16 matrix [rows, cols] (row-major), box = 64 columns (128 B, swizzled) x box_rows
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn || ptr == nullptr || (cols * 2) % 16 != 0 || rows < box_rows || cols < 64) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t gemm(const CUtensorMap& ma, const CUtensorMap& mb, const GemmParams& p,
                 cudaStream_t st) {
  const int tiles = p.batches * ((p.N + kBN - 1) / kBN) * ((p.M + kBM - 1) / kBM);
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  const size_t smem = 1024 + (size_t)kStages * kStageBytes + sizeof(SmemG);
  cudaError_t e = cudaFuncSetAttribute(k_out_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return launch(false, k_out_proj_tc, dim3(grid), dim3(kThreads), smem, st, ma, mb, p);
}

}  // namespace

bool out_proj_tc_shape_ok(const proj::Geom& G) {
  return G.Q >= kBM && G.K1 % kBK == 0 && (G.g * G.d_g) % kBK == 0 && G.d_g % 8 == 0 &&
         G.d % 8 == 0 && G.d_g >= 64 && G.d >= 64;
}

size_t out_proj_tc_workspace_bytes(const proj::Geom& G) {
  return (size_t)G.Q * G.g * G.d_g * 2 + 256;  // the bf16 intermediate
}

cudaError_t launch_out_proj_tc(const OutProjArgs& a, void* ws, cudaStream_t st) {
  const proj::Geom& G = a.G;
  __nv_bfloat16* mid = static_cast<__nv_bfloat16*>(ws);
  CUtensorMap ma1, mb1, ma2, mb2;
  memset(&ma1, 0, sizeof(ma1));
  memset(&mb1, 0, sizeof(mb1));
  memset(&ma2, 0, sizeof(ma2));
  memset(&mb2, 0, sizeof(mb2));
  const int K2 = G.g * G.d_g;
  if (!make_map(&ma1, a.o, G.Q, (uint64_t)G.H * G.c, kBM) ||
      !make_map(&mb1, a.w_grp, (uint64_t)G.g * G.K1, G.d_g, kBK) ||
      !make_map(&ma2, mid, G.Q, K2, kBM) || !make_map(&mb2, a.w_out, K2, G.d, kBK))
    return cudaErrorInvalidValue;
  GemmParams p1{G.Q, G.d_g, G.K1, G.g, G.K1, G.K1, G.d_g, K2, mid};
  cudaError_t e = gemm(ma1, mb1, p1, st);
  if (e != cudaSuccess) return e;
  GemmParams p2{G.Q, G.d, K2, 1, 0, 0, 0, G.d, a.out};
  return gemm(ma2, mb2, p2, st);
}

cudaError_t out_proj_tc_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, tc::g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));
}

}  // namespace csa
