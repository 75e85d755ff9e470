// Stage 2 on tensor cores for MXFP4 indexer keys and queries (decode).
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): I[t,s] = sum_h w[t,h] * ReLU(q^I[t,h] . K[s]);
// 二(四) FP4 量化感知训练: the indexer's QK path is cached, loaded and multiplied in FP4.
//
// One tile = 128 keys of one query's request: D[128 keys x 64 heads] = K_tile . q^T over
// d_I = 128, as two tcgen05 kind::mxf4 block-scaled MMAs (K = 64 each, one e8m0 scale per
// 32 elements of A and of B, products exact, fp32 accumulation in TMEM). TMEM lane = key,
// column = head, so each epilogue thread owns one key and reduces its 64 head dots with
// w * ReLU(.) without any shuffle.
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0  TMA producer: key tile (128 x 64 B, 64B-swizzled), its 128 scale words, the
//           query's 64 x 64 B heads and their scale words, into an 8-stage ring;
//   warp 1  MMA issuer: rearranges the scale words into the 32x128b layout tcgen05.cp
//           copies into TMEM (row 32*j + i of the tile -> lane i, column j; the 4 bytes of
//           a column are the row's 4 block scales), then issues the copy and the 2 MMAs;
//   warps 2-5 epilogue: TMEM -> registers (32x32b.x64), w * ReLU head sum, fp32 store.
// Four accumulator slots in TMEM let the MMAs of tiles j+1..j+3 run while the epilogue
// reduces tile j. Work (query, tile) pairs are split
// evenly over the CTAs; ragged per-query visibility is handled by masking the stores.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kStages = 8;
constexpr int kTileKeys = 128;     // M
constexpr int kHeads = 64;         // N (indexer heads)
constexpr int kRowBytes = 64;      // 128 e2m1 per row
constexpr int kMaxQueries = 1024;  // (request, query) pairs per launch
constexpr int kThreads = 192;

constexpr int kOffA = 0;                                 // 8192 B, 1024-aligned
constexpr int kOffQ = kOffA + kTileKeys * kRowBytes;     // 4096 B
constexpr int kOffSA = kOffQ + kHeads * kRowBytes;       // 512 B  key scale words
constexpr int kOffSQ = kOffSA + kTileKeys * 4;           // 256 B  query scale words
constexpr int kOffSFA = kOffSQ + kHeads * 4;             // 512 B  rearranged for tcgen05.cp
constexpr int kOffSFB = kOffSFA + 512;                   // 512 B
constexpr int kStageBytes = ((kOffSFB + 512 + 1023) / 1024) * 1024;
constexpr uint32_t kStageTx = kTileKeys * kRowBytes + kHeads * kRowBytes + kTileKeys * 4 +
                              kHeads * 4;

// TMEM columns
constexpr int kAcc = 4;  // accumulator slots in TMEM
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t acc_col(int acc) { return 64u * acc; }         // 0..192
__device__ __forceinline__ uint32_t sfa_col(int acc) { return 256u + 32u * acc; }  // 256..352
__device__ __forceinline__ uint32_t sfb_col(int acc) { return 272u + 32u * acc; }  // 272..368

// device error codes of this kernel
enum { kErrFull = 101, kErrEmpty = 102, kErrTmemFull = 103, kErrTmemEmpty = 104 };

struct Mxf4Params {
  int Q, T, m;
  int64_t n_cap;
  const int64_t* q_pos;
  const float* w;
  float* scores;
  int* hist;  // optional [Q][4096] histogram of the scores' top 12 key bits
};

constexpr int kBins = 4096;

struct Smem {
  uint64_t full[kStages], empty[kStages], tfull[kAcc], tempty[kAcc], done;
  uint32_t tmem_slot;
  int prefix[kMaxQueries + 1];
  int nvis[kMaxQueries];
  int hist[kBins];
};

// named barrier of the 4 epilogue warps; returns the AND of `ok` over them
__device__ __forceinline__ bool epi_all_ok(bool ok) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 2, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(res)
      : "r"((uint32_t)ok)
      : "memory");
  return res != 0;
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__device__ __forceinline__ int find_query(const int* prefix, int Q, int u) {
  int lo = 0, hi = Q;  // largest q with prefix[q] <= u
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_index_mxf4_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ks,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qs,
                    Mxf4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Smem& S = *reinterpret_cast<Smem*>(base + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- per-query visible counts and tile prefix (warp 0, warp-level scan) ----
  if (warp == 0) {
    int run = 0;
    for (int q0 = 0; q0 < p.Q; q0 += 32) {
      const int q = q0 + lane;
      int nv = 0;
      if (q < p.Q) {
        const int64_t t = p.q_pos[q];
        const int64_t v = t < 0 ? 0 : (t / p.m < p.n_cap ? t / p.m : p.n_cap);
        nv = (int)v;
        S.nvis[q] = nv;
      }
      const int tiles = (nv + kTileKeys - 1) / kTileKeys;
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      if (q < p.Q) S.prefix[q] = run + incl - tiles;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      S.prefix[p.Q] = run;
      mbar_init(&S.done, 1);
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&S.full[i], 1);
        mbar_init(&S.empty[i], 1);
      }
      for (int i = 0; i < kAcc; ++i) {
        mbar_init(&S.tfull[i], 1);
        mbar_init(&S.tempty[i], 4);
      }
      fence_barrier_init();
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_ks);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_qs);
    }
  } else if (warp == 1) {
    tmem_alloc(&S.tmem_slot, kTmemCols);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_slot;
  const int U = S.prefix[p.Q];
  const int u0 = (int)(((int64_t)U * blockIdx.x) / gridDim.x);
  const int u1 = (int)(((int64_t)U * (blockIdx.x + 1)) / gridDim.x);

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0 && u0 < u1) {
      int q = find_query(S.prefix, p.Q, u0);
      int k = 0;
      for (int u = u0; u < u1; ++u, ++k) {
        while (u >= S.prefix[q + 1]) ++q;
        const int tile = u - S.prefix[q];
        const int st = k % kStages;
        const uint32_t round = (uint32_t)(k / kStages);
        if (!mbar_wait(&S.empty[st], (round & 1) ^ 1, kErrEmpty)) break;
        uint8_t* sb = base + st * kStageBytes;
        const int b = q / p.T;
        const int32_t row0 = (int32_t)(b * p.n_cap + (int64_t)tile * kTileKeys);
        mbar_arrive_expect_tx(&S.full[st], kStageTx);
        tma_load_2d(sb + kOffA, &tm_k, 0, row0, &S.full[st]);
        tma_load_1d(sb + kOffSA, &tm_ks, row0, &S.full[st]);
        tma_load_2d(sb + kOffQ, &tm_q, 0, q * kHeads, &S.full[st]);
        tma_load_1d(sb + kOffSQ, &tm_qs, q * kHeads, &S.full[st]);
      }
      // drain: do not leave the CTA while copies into its shared memory are in flight
      const int issued = k;
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait(&S.full[j % kStages], (uint32_t)((j / kStages) & 1), kErrFull);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    const uint32_t id0 = idesc_mxf4(kTileKeys, kHeads, 0, 0);
    const uint32_t id1 = idesc_mxf4(kTileKeys, kHeads, 2, 2);
    int k = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok; ++u, ++k) {
      const int st = k % kStages;
      const uint32_t round = (uint32_t)(k / kStages);
      const int acc = k % kAcc;
      const uint32_t around = (uint32_t)(k / kAcc);
      ok = mbar_wait(&S.full[st], round & 1, kErrFull);
      if (!ok) break;
      uint8_t* sb = base + st * kStageBytes;
      // scale words -> tcgen05.cp layout: 16-byte row i = words of tile rows i, 32+i, 64+i, 96+i
      const uint32_t* sa = reinterpret_cast<const uint32_t*>(sb + kOffSA);
      const uint32_t* sq = reinterpret_cast<const uint32_t*>(sb + kOffSQ);
      *reinterpret_cast<uint4*>(sb + kOffSFA + 16 * lane) =
          make_uint4(sa[lane], sa[32 + lane], sa[64 + lane], sa[96 + lane]);
      *reinterpret_cast<uint4*>(sb + kOffSFB + 16 * lane) =
          make_uint4(sq[lane], sq[32 + lane], 0u, 0u);
      fence_proxy_async_smem();
      __syncwarp();
      int good = 1;
      if (lane == 0) {
        good = mbar_wait(&S.tempty[acc], (around & 1) ^ 1, kErrTmemEmpty);
        if (good) {
          tc_fence_after();
          const uint32_t sfa = tmem + sfa_col(acc), sfb = tmem + sfb_col(acc);
          tmem_cp_32x128b_warpx4(sfa, smem_desc(smem_u32(sb + kOffSFA), 0, 128, kLayoutNone));
          tmem_cp_32x128b_warpx4(sfb, smem_desc(smem_u32(sb + kOffSFB), 0, 128, kLayoutNone));
          const uint64_t a0 = smem_desc(smem_u32(sb + kOffA), 16, 8 * kRowBytes, kLayoutSw64);
          const uint64_t b0 = smem_desc(smem_u32(sb + kOffQ), 16, 8 * kRowBytes, kLayoutSw64);
          const uint32_t d = tmem + acc_col(acc);
          mma_mxf4(d, a0, b0, id0, sfa, sfb, 0u);
          // second K half: +32 bytes inside the swizzled rows, scale bytes 2..3
          mma_mxf4(d, a0 + 2, b0 + 2, id1, sfa | (2u << 30), sfb | (2u << 30), 1u);
          mma_commit(&S.empty[st]);
          mma_commit(&S.tfull[acc]);
        }
      }
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
    }
    // every MMA / copy this thread issued has completed once `done` fires
    if (lane == 0) {
      mma_commit(&S.done);
      mbar_wait(&S.done, 0, kErrTmemFull);
    }
    __syncwarp();
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int etid = threadIdx.x - 64;
    const bool hist = p.hist != nullptr;
    if (hist) {
      for (int i = etid; i < kBins; i += 128) S.hist[i] = 0;
      epi_bar();
    }
    int hq = -1;
    auto flush = [&](int qq) {  // smem histogram of query qq -> global, then clear
      epi_bar();
      for (int i = etid; i < kBins; i += 128) {
        const int v = S.hist[i];
        if (v) {
          atomicAdd(&p.hist[(size_t)qq * kBins + i], v);
          S.hist[i] = 0;
        }
      }
      epi_bar();
    };
    float wr[kHeads];
    int cur_q = -1;
    int q = u0 < u1 ? find_query(S.prefix, p.Q, u0) : 0;
    int k = 0;
    for (int u = u0; u < u1; ++u, ++k) {
      while (u >= S.prefix[q + 1]) ++q;
      const int tile = u - S.prefix[q];
      if (q != cur_q) {
#pragma unroll
        for (int h = 0; h < kHeads; ++h) wr[h] = p.w[(size_t)q * kHeads + h];
        cur_q = q;
      }
      if (hist && q != hq) {
        if (hq >= 0) flush(hq);
        hq = q;
      }
      const int acc = k % kAcc;
      const uint32_t around = (uint32_t)(k / kAcc);
      if (!epi_all_ok(mbar_wait(&S.tfull[acc], around & 1, kErrTmemFull))) break;
      tc_fence_after();
      uint32_t v[kHeads];
      tmem_ld_32x32b_x64(tmem + ((uint32_t)(32 * quad) << 16) + acc_col(acc), v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.tempty[acc]);
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < kHeads; ++h) sc = fmaf(wr[h], fmaxf(__uint_as_float(v[h]), 0.f), sc);
      const int s = tile * kTileKeys + 32 * quad + lane;
      if (s < S.nvis[q]) {
        p.scores[(size_t)q * p.n_cap + s] = sc;
        if (hist) atomicAdd(&S.hist[float_key(sc) >> 20], 1);
      }
    }
    if (hist && hq >= 0) flush(hq);
  }
  // ---- teardown: the MMA warp saw its last MMA complete; free TMEM ----
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host: tensor maps ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kRowBytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
  cuuint32_t box[2] = {(cuuint32_t)kRowBytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_1d_words(CUtensorMap* m, const void* ptr, uint64_t words, uint32_t box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[1] = {(cuuint64_t)words};
  cuuint64_t strides[1] = {0};
  cuuint32_t bx[1] = {box};
  cuuint32_t es[1] = {1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, const_cast<void*>(ptr), dims, strides, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

bool index_mxf4_tc_supported(const IndexArgs& a) {
  return a.kdt == CSA_MXFP4 && a.n_idx_heads == kHeads && a.d_idx == 128 && a.n_cap % 32 == 0 &&
         (int64_t)a.B * a.T <= kMaxQueries && (int64_t)a.B * a.n_cap < (1ll << 31);
}

cudaError_t launch_index_mxf4_tc(const IndexArgs& a, cudaStream_t st) {
  const int Q = a.B * a.T;
  CUtensorMap mk, mks, mq, mqs;
  if (!make_map_2d(&mk, a.KI, (uint64_t)a.B * a.n_cap, kTileKeys) ||
      !make_map_1d_words(&mks, a.KI_scale, (uint64_t)a.B * a.n_cap, kTileKeys) ||
      !make_map_2d(&mq, a.qI, (uint64_t)Q * kHeads, kHeads) ||
      !make_map_1d_words(&mqs, a.qI_scale, (uint64_t)Q * kHeads, kHeads))
    return cudaErrorInvalidValue;
  Mxf4Params p{Q, a.T, a.m, a.n_cap, a.q_pos, a.w, a.scores, a.hist};
  const int64_t units_max = (int64_t)Q * ((a.n_cap + kTileKeys - 1) / kTileKeys);
  const int grid = (int)(units_max < num_sms() ? (units_max > 0 ? units_max : 1) : num_sms());
  const size_t smem = 1024 + (size_t)kStages * kStageBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(k_index_mxf4_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  timing_before(st);
  k_index_mxf4_tc<<<grid, kThreads, smem, st>>>(mk, mks, mq, mqs, p);
  timing_after(st);
  return cudaGetLastError();
}

cudaError_t index_mxf4_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, tc::g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));
}

}  // namespace csa
