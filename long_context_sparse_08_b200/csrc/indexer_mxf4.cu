// Stage 2 on tensor cores for MXFP4 indexer keys and queries (decode).
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): I[t,s] = sum_h w[t,h] * ReLU(q^I[t,h] . K[s]);
// 二(四) FP4 量化感知训练: the indexer's QK path is cached, loaded and multiplied in FP4.
//
// A unit is 512 keys of one query's request: four M-tiles of 128 keys, each
// D[128 keys x 64 heads] = K_tile . q^T over d_I = 128 as two tcgen05 kind::mxf4
// block-scaled MMAs (K = 64 each, one e8m0 scale per 32 elements of A and of B, exact
// products, fp32 accumulation in TMEM). TMEM lane = key, column = head, so an epilogue
// thread owns one key and reduces its 64 head dots with w * ReLU(.) without shuffles.
//
// Key scales are stored in 128-key blocks laid out as tcgen05.cp's 32x128b source: byte
// 16*i + 4*j + b of a block is block-scale b of key 32*j + i. One TMA copy of a unit's
// 2 KB of scales therefore lands ready for tcgen05.cp (no rearrangement in the kernel).
//
// Persistent kernel, one CTA per SM, 11 warps:
//   warp 0     TMA producer: per unit one 32 KB key box (64B-swizzled) and one 2 KB scale
//              box; per query the 64 x 64 B heads and their scale words;
//   warps 1,10 MMA issuers (one lane each): warp 1 takes M-tiles 0-1 of every unit, warp 10
//              M-tiles 2-3, each into its own TMEM slot; per query each copies the query
//              scales into its own TMEM columns, per M-tile the key scales (tcgen05.cp),
//              then two MMAs. An MMA of this shape costs the tensor unit ~50 cycles however
//              many threads issue, but the copies, waits and commits cost the issuing
//              thread; two issuers run those chains side by side;
//   warps 2-9  two epilogue warpgroups; group g reduces M-tiles g and 2 + g of each unit:
//              TMEM -> registers, w * ReLU head sum, fp32 score store, and a 4096-bin
//              histogram of the scores' top 12 key bits for the top-k selector.
// TMEM holds two half-unit slots (2 M-tiles each), one per issuer: while both groups
// reduce one half-unit the other issuer's MMAs run. Descriptors are precomputed and each
// issuer waits once per unit for its slot.
// Units are split evenly over the CTAs; ragged per-query visibility is handled by masking
// the stores.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kStages = 5;
constexpr int kTileKeys = 128;     // M of one MMA
constexpr int kUnitTiles = 4;
constexpr int kUnitKeys = kUnitTiles * kTileKeys;  // keys per pipeline stage
constexpr int kHeads = 64;         // N (indexer heads)
constexpr int kRowBytes = 64;      // 128 e2m1 per row
constexpr int kMaxQueries = 1024;  // (request, query) pairs per launch
constexpr int kThreads = 352;
constexpr int kWarpMma1 = kThreads / 32 - 1;  // second MMA issuer (last warp)
constexpr int kBins = 4096;

constexpr int kOffA = 0;                                // 32 KB, 1024-aligned
constexpr int kOffSF = kOffA + kUnitKeys * kRowBytes;   // 2 KB key scales (cp layout)
constexpr int kStageBytes = ((kOffSF + kUnitKeys * 4 + 1023) / 1024) * 1024;
constexpr uint32_t kStageTx = kUnitKeys * kRowBytes + kUnitKeys * 4;
// per-query buffers (two slots)
constexpr int kOffQ = 0;                                // 4 KB q heads (64B-swizzled)
constexpr int kOffQS = kOffQ + kHeads * kRowBytes;      // 256 B query scale words
constexpr int kOffQSF = kOffQS + kHeads * 4;            // 512 B rearranged for tcgen05.cp
constexpr int kQBytes = ((kOffQSF + 2 * 512 + 1023) / 1024) * 1024;  // one layout per issuer
constexpr uint32_t kQTx = kHeads * kRowBytes + kHeads * 4;

// TMEM columns: two half-unit slots of two 64-column accumulators, their key-scale columns,
// two query-scale slots
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t acc_col(int hs, int j) { return 128u * hs + 64u * j; }
__device__ __forceinline__ uint32_t sfa_col(int hs, int j) { return 256u + 16u * hs + 8u * j; }
__device__ __forceinline__ uint32_t sfb_col(int qs, int h) { return 288u + 16u * qs + 8u * h; }

enum { kErrFull = 101, kErrEmpty = 102, kErrTmemFull = 103, kErrTmemEmpty = 104,
       kErrQFull = 105, kErrQEmpty = 106, kErrPageId = 107 };

struct Mxf4Params {
  int Q, T, m;
  int64_t n_cap;
  const int64_t* q_pos;
  const float* w;
  float* scores;
  int* hist;  // optional [Q][4096] histogram of the scores' top 12 key bits
};

// The variants' extra inputs (a separate kernel parameter, so the plain kernel's stays as is)
struct Mxf4Ext {
  __nv_bfloat16* scores16;    // kB16: the scores rounded once to bf16, stored instead
  const int32_t* page_table;  // kPaged: keys and their scale blocks in a page pool; key e of
                              // request b is row e % page_rows of page
                              // page_table[b * max_pages + e / page_rows]
  int page_rows, max_pages, n_pages;  // page_rows a multiple of 128
};

struct Smem {
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], qfull[2], qempty[2], done;
  uint32_t tmem_slot;
  int prefix[kMaxQueries + 1];
  int nvis[kMaxQueries];
  int hist[kBins];
};

__device__ __forceinline__ int find_query(const int* prefix, int Q, int u) {
  int lo = 0, hi = Q;  // largest q with prefix[q] <= u
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid;
  }
  return lo;
}

// named barrier 2 over the 8 epilogue warps; returns the AND of `ok` over them
__device__ __forceinline__ bool epi_all_ok(bool ok) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 2, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(res)
      : "r"((uint32_t)ok)
      : "memory");
  return res != 0;
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 2, 256;" ::: "memory"); }

// The kernel body. kPaged: each 128-key block of a unit is its own TMA box, read through the
// page table (tm_k / tm_ks then cover the pool with one-block boxes); a block past the
// query's visible keys reads pool block 0 and is masked like any invisible key, and a page id
// outside the pool records kErrPageId and reads block 0. kB16: bf16 score stores.
template <bool kPaged, bool kB16>
__device__ __forceinline__ void index_mxf4_body(const CUtensorMap& tm_k, const CUtensorMap& tm_ks,
                                                const CUtensorMap& tm_q, const CUtensorMap& tm_qs,
                                                const Mxf4Params& p, const Mxf4Ext& x) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  uint8_t* qbase = base + kStages * kStageBytes;
  Smem& S = *reinterpret_cast<Smem*>(qbase + 2 * kQBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- set-up that reads nothing a predecessor writes: barriers, TMEM, descriptors ----
  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&S.full[i], 1);
        mbar_init(&S.empty[i], 2);  // both issuers' MMAs read the stage
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&S.tfull[i], 1);
        mbar_init(&S.tempty[i], 8);  // every epilogue warp
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&S.qfull[i], 1);
        mbar_init(&S.qempty[i], 2);
      }
      mbar_init(&S.done, 2);
      fence_barrier_init();
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_ks);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_qs);
    }
  } else if (warp == 1) {
    tmem_alloc(&S.tmem_slot, kTmemCols);
  } else if (warp != kWarpMma1) {
    for (int i = threadIdx.x - 64; i < kBins; i += 256) S.hist[i] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // positions, scores and the histogram belong to the previous kernels from here on
  pdl_wait();
  pdl_trigger();
  // ---- per-query visible counts and unit prefix (warp 0, warp-level scan) ----
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
      const int units = (nv + kUnitKeys - 1) / kUnitKeys;
      int incl = units;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      if (q < p.Q) S.prefix[q] = run + incl - units;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) S.prefix[p.Q] = run;
  }
  __syncthreads();
  const uint32_t tmem = S.tmem_slot;
  const int U = S.prefix[p.Q];
  const int u0 = (int)(((int64_t)U * blockIdx.x) / gridDim.x);
  const int u1 = (int)(((int64_t)U * (blockIdx.x + 1)) / gridDim.x);

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0 && u0 < u1) {
      int q = find_query(S.prefix, p.Q, u0);
      int cur_q = -1, nq = -1;  // nq: index of the current query within this CTA
      int k = 0, issued_q = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u, ++k) {
        while (u >= S.prefix[q + 1]) ++q;
        if (q != cur_q) {  // this query's heads and their scale words into the next slot
          ++nq;
          cur_q = q;
          const int qs = nq & 1;
          ok = mbar_wait(&S.qempty[qs], ((nq >> 1) & 1) ^ 1, kErrQEmpty);
          if (!ok) break;
          uint8_t* qb = qbase + qs * kQBytes;
          mbar_arrive_expect_tx(&S.qfull[qs], kQTx);
          tma_load_2d(qb + kOffQ, &tm_q, 0, q * kHeads, &S.qfull[qs]);
          tma_load_1d(qb + kOffQS, &tm_qs, q * kHeads, &S.qfull[qs]);
          issued_q = nq + 1;
        }
        const int unit = u - S.prefix[q];
        const int st = k % kStages;
        const uint32_t round = (uint32_t)(k / kStages);
        ok = mbar_wait(&S.empty[st], (round & 1) ^ 1, kErrEmpty);
        if (!ok) break;
        uint8_t* sb = base + st * kStageBytes;
        const int b = q / p.T;
        if constexpr (kPaged) {
          mbar_arrive_expect_tx(&S.full[st], kStageTx);
#pragma unroll 1
          for (int j = 0; j < kUnitTiles; ++j) {
            const int64_t e = (int64_t)unit * kUnitKeys + j * kTileKeys;  // block's first key
            int32_t blk = 0;
            if (e < S.nvis[q]) {
              const int32_t pg = x.page_table[(size_t)b * x.max_pages + e / x.page_rows];
              if (pg >= 0 && pg < x.n_pages)
                blk = (int32_t)(((int64_t)pg * x.page_rows + e % x.page_rows) / kTileKeys);
              else
                set_error(kErrPageId);
            }
            tma_load_3d(sb + kOffA + j * (kTileKeys * kRowBytes), &tm_k, 0, 0, blk, &S.full[st]);
            tma_load_2d(sb + kOffSF + j * (kTileKeys * 4), &tm_ks, 0, blk, &S.full[st]);
          }
        } else {
          // keys and scales are viewed in 128-key blocks; a unit is 4 consecutive blocks
          const int32_t blk0 =
              (int32_t)((b * p.n_cap + (int64_t)unit * kUnitKeys) / kTileKeys);
          mbar_arrive_expect_tx(&S.full[st], kStageTx);
          tma_load_3d(sb + kOffA, &tm_k, 0, 0, blk0, &S.full[st]);
          tma_load_2d(sb + kOffSF, &tm_ks, 0, blk0, &S.full[st]);
        }
      }
      // drain: no copy into this CTA's shared memory may still be in flight at exit
      for (int j = (k > kStages ? k - kStages : 0); j < k; ++j)
        mbar_wait(&S.full[j % kStages], (uint32_t)((j / kStages) & 1), kErrFull);
      for (int j = (issued_q > 2 ? issued_q - 2 : 0); j < issued_q; ++j)
        mbar_wait(&S.qfull[j & 1], (uint32_t)((j >> 1) & 1), kErrQFull);
    }
  } else if (warp == 1 || warp == kWarpMma1) {
    // ------------------------- MMA issuers (one lane each) -------------------------
    const int h = warp == 1 ? 0 : 1;  // this issuer's half of every unit and TMEM slot
    if (lane == 0) {
      const uint32_t id0 = idesc_mxf4(kTileKeys, kHeads, 0, 0);
      const uint32_t id1 = idesc_mxf4(kTileKeys, kHeads, 2, 2);
      const uint64_t a_desc0 = smem_desc(smem_u32(base + kOffA), 16, 8 * kRowBytes, kLayoutSw64);
      const uint64_t sf_desc0 = smem_desc(smem_u32(base + kOffSF), 0, 128, kLayoutNone);
      const uint64_t q_desc0 = smem_desc(smem_u32(qbase + kOffQ), 16, 8 * kRowBytes, kLayoutSw64);
      int q = u0 < u1 ? find_query(S.prefix, p.Q, u0) : 0;
      int cur_q = -1, nq = -1;
      int k = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u, ++k) {
        while (u >= S.prefix[q + 1]) ++q;
        if (q != cur_q) {
          if (cur_q >= 0) mma_commit(&S.qempty[nq & 1]);  // old slot free once its MMAs end
          ++nq;
          cur_q = q;
          const int qs = nq & 1;
          ok = mbar_wait(&S.qfull[qs], (nq >> 1) & 1, kErrQFull);
          if (!ok) break;
          // query scale words -> tcgen05.cp layout (16-byte row i: words of heads i, 32+i),
          // one copy per issuer
          uint8_t* qb = qbase + qs * kQBytes;
          const uint32_t* sq = reinterpret_cast<const uint32_t*>(qb + kOffQS);
          uint8_t* qsf = qb + kOffQSF + 512 * h;
          for (int i = 0; i < 32; ++i)
            *reinterpret_cast<uint4*>(qsf + 16 * i) = make_uint4(sq[i], sq[32 + i], 0u, 0u);
          fence_proxy_async_smem();
          tc_fence_after();
          tmem_cp_32x128b_warpx4(tmem + sfb_col(qs, h),
                                 smem_desc(smem_u32(qsf), 0, 128, kLayoutNone));
        }
        const int qs = nq & 1;
        const int st = k % kStages;
        ok = mbar_wait(&S.full[st], (uint32_t)(k / kStages) & 1, kErrFull);
        if (!ok) break;
        const uint64_t a_st = a_desc0 + (uint64_t)st * (kStageBytes >> 4);
        const uint64_t sf_st = sf_desc0 + (uint64_t)st * (kStageBytes >> 4);
        const uint64_t b0 = q_desc0 + (uint64_t)qs * (kQBytes >> 4);
        const uint32_t sfb = tmem + sfb_col(qs, h);
        ok = mbar_wait(&S.tempty[h], ((uint32_t)k & 1) ^ 1, kErrTmemEmpty);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 2; ++j)  // key scales of both tiles first (latencies overlap)
          tmem_cp_32x128b_warpx4(tmem + sfa_col(h, j), sf_st + (uint64_t)(2 * h + j) * 32);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint64_t a0 = a_st + (uint64_t)(2 * h + j) * 512;  // 8 KB per M-tile
          const uint32_t d = tmem + acc_col(h, j), sfa = tmem + sfa_col(h, j);
          mma_mxf4(d, a0, b0, id0, sfa, sfb, 0u);
          // second K half: +32 bytes inside the swizzled rows, scale bytes 2..3
          mma_mxf4(d, a0 + 2, b0 + 2, id1, sfa | (2u << 30), sfb | (2u << 30), 1u);
        }
        mma_commit(&S.tfull[h]);
        mma_commit(&S.empty[st]);
      }
      // every MMA / copy this thread issued has completed once `done` fires (both issuers)
      mma_commit(&S.done);
      mbar_wait(&S.done, 0, kErrTmemFull);
    }
    __syncwarp();
  } else {
    // ------------------------------ epilogue ------------------------------
    const int grp = (warp - 2) >> 2;  // M-tile this warpgroup reduces
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const bool hist = p.hist != nullptr;
    int hq = -1;
    auto flush = [&](int qq) {  // shared histogram of query qq -> global, then clear
      epi_bar();
      for (int i = threadIdx.x - 64; i < kBins; i += 256) {
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
    bool ok = true;
    for (int u = u0; u < u1 && ok; ++u, ++k) {
      while (u >= S.prefix[q + 1]) ++q;
      const int unit = u - S.prefix[q];
      if (q != cur_q) {
#pragma unroll
        for (int h = 0; h < kHeads; ++h) wr[h] = p.w[(size_t)q * kHeads + h];
        cur_q = q;
      }
      if (hist && q != hq) {
        if (hq >= 0) flush(hq);
        hq = q;
      }
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {  // this group reduces M-tile 2h + grp of the unit
        const int n = 2 * k + h, hs = n & 1, t = 2 * h + grp;
        ok = epi_all_ok(mbar_wait(&S.tfull[hs], (uint32_t)(n >> 1) & 1, kErrTmemFull));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[kHeads];
        tmem_ld_32x32b_x64(tmem + ((uint32_t)(32 * quad) << 16) + acc_col(hs, grp), v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.tempty[hs]);
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh)
          part[hh & 3] = fmaf(wr[hh], fmaxf(__uint_as_float(v[hh]), 0.f), part[hh & 3]);
        const float sc = (part[0] + part[1]) + (part[2] + part[3]);
        const int s = unit * kUnitKeys + t * kTileKeys + 32 * quad + lane;
        if (s < S.nvis[q]) {
          if constexpr (kB16) {  // BF16 index scores: round once, select on the rounded value
            const __nv_bfloat16 r = __float2bfloat16_rn(sc);
            x.scores16[(size_t)q * p.n_cap + s] = r;
            if (hist) atomicAdd(&S.hist[float_key(__bfloat162float(r)) >> 20], 1);
          } else {
            p.scores[(size_t)q * p.n_cap + s] = sc;
            if (hist) atomicAdd(&S.hist[float_key(sc) >> 20], 1);
          }
        }
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

__global__ void __launch_bounds__(kThreads, 1)
    k_index_mxf4_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ks,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qs,
                    Mxf4Params p) {
  index_mxf4_body<false, false>(tm_k, tm_ks, tm_q, tm_qs, p, Mxf4Ext{});
}

// paged keys and / or BF16 index scores
template <bool kPaged, bool kB16>
__global__ void __launch_bounds__(kThreads, 1)
    k_index_mxf4_ext(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ks,
                     const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qs,
                     Mxf4Params p, Mxf4Ext x) {
  index_mxf4_body<kPaged, kB16>(tm_k, tm_ks, tm_q, tm_qs, p, x);
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

// keys as [128-key blocks][128 rows][64 B], box = `blocks` blocks (4: one 512-key unit;
// 1: one block, for page pools)
bool make_map_keys(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t blocks) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kRowBytes, (cuuint64_t)kTileKeys,
                        (cuuint64_t)(rows / kTileKeys)};
  cuuint64_t strides[2] = {(cuuint64_t)kRowBytes, (cuuint64_t)kRowBytes * kTileKeys};
  cuuint32_t box[3] = {(cuuint32_t)kRowBytes, (cuuint32_t)kTileKeys, blocks};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// key scale words as [128-key blocks][128 words], box = `blocks` blocks
bool make_map_key_scales(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t blocks) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kTileKeys, (cuuint64_t)(rows / kTileKeys)};
  cuuint64_t strides[1] = {(cuuint64_t)kTileKeys * 4};
  cuuint32_t box[2] = {(cuuint32_t)kTileKeys, blocks};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  const bool rows_ok = a.page_table == nullptr
                           ? (int64_t)a.B * a.n_cap < (1ll << 31)
                           : a.page_rows > 0 && a.page_rows % kTileKeys == 0 && a.n_pages > 0 &&
                                 (int64_t)a.n_pages * a.page_rows < (1ll << 31);
  return a.kdt == CSA_MXFP4 && a.n_idx_heads == kHeads && a.d_idx == 128 && a.n_cap % 128 == 0 &&
         (int64_t)a.B * a.T <= kMaxQueries && rows_ok;
}

namespace {
template <bool kPaged, bool kB16>
cudaError_t launch_ext(const CUtensorMap& mk, const CUtensorMap& mks, const CUtensorMap& mq,
                       const CUtensorMap& mqs, const Mxf4Params& p, const Mxf4Ext& x, int grid,
                       size_t smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(k_index_mxf4_ext<kPaged, kB16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch(true, k_index_mxf4_ext<kPaged, kB16>, dim3(grid), dim3(kThreads), smem, st, mk,
                mks, mq, mqs, p, x);
}
}  // namespace

cudaError_t launch_index_mxf4_tc(const IndexArgs& a, cudaStream_t st) {
  const int Q = a.B * a.T;
  const bool paged = a.page_table != nullptr, b16 = a.scores16 != nullptr;
  // keys: the contiguous cache [B, n_cap] in 4-block boxes, or the pool in 1-block boxes
  const uint64_t key_rows = paged ? (uint64_t)a.n_pages * a.page_rows : (uint64_t)a.B * a.n_cap;
  const uint32_t blocks = paged ? 1u : (uint32_t)kUnitTiles;
  CUtensorMap mk, mks, mq, mqs;
  if (!make_map_keys(&mk, a.KI, key_rows, blocks) ||
      !make_map_key_scales(&mks, a.KI_scale, key_rows, blocks) ||
      !make_map_2d(&mq, a.qI, (uint64_t)Q * kHeads, kHeads) ||
      !make_map_1d_words(&mqs, a.qI_scale, (uint64_t)Q * kHeads, kHeads))
    return cudaErrorInvalidValue;
  Mxf4Params p{Q, a.T, a.m, a.n_cap, a.q_pos, a.w, a.scores, a.hist};
  const int64_t units_max = (int64_t)Q * ((a.n_cap + kUnitKeys - 1) / kUnitKeys);
  const int grid = (int)(units_max < num_sms() ? (units_max > 0 ? units_max : 1) : num_sms());
  const size_t smem = 1024 + (size_t)kStages * kStageBytes + 2 * kQBytes + sizeof(Smem);
  if (paged || b16) {
    const Mxf4Ext x{static_cast<__nv_bfloat16*>(a.scores16), a.page_table, a.page_rows,
                    a.max_pages, a.n_pages};
    timing_before(st);
    const cudaError_t e =
        paged ? (b16 ? launch_ext<true, true>(mk, mks, mq, mqs, p, x, grid, smem, st)
                     : launch_ext<true, false>(mk, mks, mq, mqs, p, x, grid, smem, st))
              : launch_ext<false, true>(mk, mks, mq, mqs, p, x, grid, smem, st);
    timing_after(st);
    return e;
  }
  cudaError_t e = cudaFuncSetAttribute(k_index_mxf4_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  timing_before(st);
  // programmatic launch always: the set-up before its wait reads no predecessor's data
  e = launch(true, k_index_mxf4_tc, dim3(grid), dim3(kThreads), smem, st, mk, mks, mq, mqs, p);
  timing_after(st);
  return e;
}

cudaError_t index_mxf4_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, tc::g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));
}

}  // namespace csa
