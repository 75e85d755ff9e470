// Stage 2 on tensor cores for FP8 (e4m3 + row scale) and bf16 indexer keys with bf16
// queries (decode).
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): I[t,s] = sum_h w[t,h] * ReLU(q^I[t,h] . K[s]).
//
// A tile is 128 keys of one query's request: D[128 keys x 64 heads] = K_tile . q^T over
// d_I = 128 as eight tcgen05 kind::f16 MMAs (K = 16 each, bf16 operands, fp32 accumulation
// in TMEM). TMEM lane = key, so an epilogue thread owns one key and reduces its 64 head
// dots with w * ReLU(.) without shuffles.
//
// FP8 keys: an e4m3 code is exactly a bf16 value, so converter warps rewrite each staged
// 16 KB tile of codes as the 32 KB bf16 operand (128B-swizzled, K-major); the row scale is
// positive and commutes with ReLU, so the epilogue multiplies it into the finished sum (the
// same order as the CUDA-core kernel). bf16 keys: TMA writes the operand tile directly.
//
// Prefill (bf16 keys, several queries per request): four consecutive queries of a request
// share every key tile, so one MMA is N = 256 (4 x 64 heads). An f16 MMA of N = 64 costs the
// tensor unit several times its arithmetic; at N = 256 the arithmetic dominates.
//
// Persistent kernel, one CTA per SM, 10 warps:
//   warp 0     TMA producer: per tile the key codes (fp8: into a staging ring; bf16: into
//              the operand ring), per query group the heads of q^I (two 128B-swizzled boxes);
//   warp 1     MMA issuer (one lane);
//   warps 2-5  converters (fp8 only): staging -> bf16 operand tile; with query groups of
//              four they are a second epilogue group instead;
//   warps 6-9  epilogue: TMEM -> registers, w * ReLU head sum, times the row scale (fp8),
//              fp32 score store, 4096-bin histogram of the scores' top 12 key bits (one
//              query per tile only).
// Tiles are split evenly over the CTAs; ragged visibility is handled by masking the stores.
#include <cudaTypedefs.h>


#include "common.cuh"
#include "host_util.cuh"
#include "internal.h"
#include "tc.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kTileKeys = 128;    // M of one MMA
constexpr int kHeads = 64;        // indexer heads (N of one query)
constexpr int kDim = 128;         // d_I
constexpr int kMaxQueries = 512;  // (request, query) pairs per launch
constexpr int kThreads = 320;
constexpr int kBins = 4096;
constexpr int kStg = 4;           // fp8 staging tiles (16 KB of codes each)

constexpr int kStgBytes = kTileKeys * kDim;         // 16 KB of e4m3 codes
constexpr int kOpBytes = kTileKeys * kDim * 2;      // 32 KB: 2 atoms x 128 rows x 128 B
constexpr int kAtomBytes = kTileKeys * 128;         // 16 KB
constexpr int kQBytes = kHeads * kDim * 2;          // 16 KB per query: 2 atoms x 64 x 128 B

enum { kErrStgFull = 301, kErrStgEmpty = 302, kErrOpFull = 303, kErrOpEmpty = 304,
       kErrTFull = 305, kErrTEmpty = 306, kErrQFull = 307, kErrQEmpty = 308, kErrPageId = 309 };

// G consecutive queries of one request share each key tile: N = 64 G per MMA.
template <bool kFp8, int G>
struct Cfg {
  static constexpr int kQSlots = G == 1 ? 2 : 1;      // q tiles in flight
  static constexpr int kOpN = kFp8 ? 3 : (G == 1 ? 5 : 4);
  static constexpr int kAccN = G == 1 ? 4 : 2;        // TMEM accumulator slots
  static constexpr int kAccCols = 64 * G;
  static constexpr int kTmemCols = kAccN * kAccCols;  // 256 or 512
  static constexpr int kQSlotBytes = G * kQBytes;
  static constexpr int kQAtomBytes = G * kHeads * 128;
  static constexpr int kEpiWarps = G == 1 ? 4 : 8;    // warps 6-9, or 2-9
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kEpiWarp0 = 10 - kEpiWarps;
  static constexpr bool kHist = G == 1;
};

struct Bf16IdxParams {
  int Q, T, m;
  int q0;  // global index of this launch's first query (launches take <= kMaxQueries)
  int64_t n_cap;
  const int64_t* q_pos;
  const float* w;
  const float* key_scale;  // fp8: [B * n_cap] row scales; bf16: nullptr
  float* scores;
  int* hist;  // optional [Q][4096]
  __nv_bfloat16* scores16;  // kB16: scores rounded to bf16 (the selector reads these)
  const int32_t* page_table;  // kPaged: keys (and FP8 row scales) in a page pool
  int page_rows, max_pages, n_pages;
};

// Row of key e of request b in the key rows the tensor map covers: contiguous [B, n_cap], or
// (kPaged) the page pool through the page table. A page id outside the pool records an
// error and reads row 0 (that tile's scores are then meaningless).
template <bool kPaged>
__device__ __forceinline__ int64_t key_row(const Bf16IdxParams& p, int b, int64_t e) {
  if constexpr (kPaged) {
    const int32_t pg = p.page_table[(size_t)b * p.max_pages + e / p.page_rows];
    if (pg < 0 || pg >= p.n_pages) {
      tc::set_error(kErrPageId);
      return 0;
    }
    return (int64_t)pg * p.page_rows + e % p.page_rows;
  } else {
    return (int64_t)b * p.n_cap + e;
  }
}

template <bool kHist>
struct Smem {
  uint64_t stg_full[kStg], stg_empty[kStg], op_full[5], op_empty[5];
  uint64_t tfull[4], tempty[4], qfull[2], qempty[2], done;
  uint32_t tmem_slot;
  int ngroups;
  int prefix[kMaxQueries + 1];  // tile prefix over groups
  int gfirst[kMaxQueries];      // first (local) query of each group
  int nvis[kMaxQueries];        // visible entries of each query
  float wst[4][kHeads];         // head weights of the current group (G > 1)
  int hist[kHist ? kBins : 1];
};

__device__ __forceinline__ int find_group(const int* prefix, int ng, int u) {
  int lo = 0, hi = ng;  // largest g with prefix[g] <= u
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid;
  }
  return lo;
}

// AND of `ok` over the kN threads of named barrier kId
template <int kId, int kN>
__device__ __forceinline__ bool group_all_ok(bool ok) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(res)
      : "r"((uint32_t)ok), "n"(kId), "n"(kN)
      : "memory");
  return res != 0;
}
template <int kN>
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 2, %0;" ::"n"(kN) : "memory");
}

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// two e4m3 codes (low byte = first) -> bf16x2, exact
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
  const __half2 hh = *reinterpret_cast<const __half2*>(&h2);
  const float2 f = __half22float2(hh);
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

template <bool kFp8, int G, bool kB16, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
    k_index_bf16_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                    Bf16IdxParams p) {
  using C = Cfg<kFp8, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  uint8_t* opbase = base;                               // kOpN x 32 KB
  uint8_t* qbase = opbase + C::kOpN * kOpBytes;         // kQSlots x G x 16 KB
  uint8_t* stgbase = qbase + C::kQSlots * C::kQSlotBytes;  // fp8: kStg x 16 KB
  Smem<C::kHist>& S =
      *reinterpret_cast<Smem<C::kHist>*>(stgbase + (kFp8 ? kStg * kStgBytes : 0));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- set-up that reads nothing a predecessor writes ----
  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kStg; ++i) {
        mbar_init(&S.stg_full[i], 1);
        mbar_init(&S.stg_empty[i], 128);
      }
      for (int i = 0; i < C::kOpN; ++i) {
        mbar_init(&S.op_full[i], kFp8 ? 128 : 1);
        mbar_init(&S.op_empty[i], 1);
      }
      for (int i = 0; i < C::kAccN; ++i) {
        mbar_init(&S.tfull[i], 1);
        mbar_init(&S.tempty[i], C::kEpiWarps);
      }
      for (int i = 0; i < C::kQSlots; ++i) {
        mbar_init(&S.qfull[i], 1);
        mbar_init(&S.qempty[i], 1);
      }
      mbar_init(&S.done, 1);
      fence_barrier_init();
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_q);
    }
  } else if (warp == 1) {
    tmem_alloc(&S.tmem_slot, C::kTmemCols);
  } else if (C::kHist && warp >= C::kEpiWarp0) {
    for (int i = threadIdx.x - 32 * C::kEpiWarp0; i < kBins; i += C::kEpiThreads) S.hist[i] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();
  // ---- groups (G consecutive queries of one request) and their tile prefix (warp 0) ----
  if (warp == 0) {
    int ng = 0;
    for (int qb0 = 0; qb0 < p.Q; qb0 += 32) {
      const int q = qb0 + lane;
      bool start = false;
      if (q < p.Q) {
        const int64_t t = p.q_pos[q];
        const int64_t v = t < 0 ? 0 : (t / p.m < p.n_cap ? t / p.m : p.n_cap);
        S.nvis[q] = (int)v;
        start = q == 0 || ((p.q0 + q) % p.T) % G == 0;
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, start);
      if (start) S.gfirst[ng + __popc(bal & ((1u << lane) - 1u))] = q;
      ng += __popc(bal);
    }
    __syncwarp();
    int run = 0;
    for (int g0 = 0; g0 < ng; g0 += 32) {
      const int g = g0 + lane;
      int tiles = 0;
      if (g < ng) {
        const int f = S.gfirst[g], e = g + 1 < ng ? S.gfirst[g + 1] : p.Q;
        int nv = 0;
        for (int mq = f; mq < e; ++mq) nv = max(nv, S.nvis[mq]);
        tiles = (nv + kTileKeys - 1) / kTileKeys;
      }
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      if (g < ng) S.prefix[g] = run + incl - tiles;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      S.prefix[ng] = run;
      S.ngroups = ng;
    }
  }
  __syncthreads();
  const uint32_t tmem = S.tmem_slot;
  const int NG = S.ngroups;
  const int U = S.prefix[NG];
  const int u0 = (int)(((int64_t)U * blockIdx.x) / gridDim.x);
  const int u1 = (int)(((int64_t)U * (blockIdx.x + 1)) / gridDim.x);
  auto gsize = [&](int g) { return (g + 1 < NG ? S.gfirst[g + 1] : p.Q) - S.gfirst[g]; };

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0 && u0 < u1) {
      int g = find_group(S.prefix, NG, u0);
      int cur_g = -1, ng = -1, k = 0, issued_q = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u, ++k) {
        while (u >= S.prefix[g + 1]) ++g;
        if (g != cur_g) {  // this group's q^I heads into the next q slot
          ++ng;
          cur_g = g;
          const int qs = ng % C::kQSlots;
          ok = mbar_wait(&S.qempty[qs], ((ng / C::kQSlots) & 1) ^ 1, kErrQEmpty);
          if (!ok) break;
          uint8_t* qb = qbase + qs * C::kQSlotBytes;
          mbar_arrive_expect_tx(&S.qfull[qs], C::kQSlotBytes);
          tma_load_2d(qb, &tm_q, 0, S.gfirst[g] * kHeads, &S.qfull[qs]);
          tma_load_2d(qb + C::kQAtomBytes, &tm_q, 64, S.gfirst[g] * kHeads, &S.qfull[qs]);
          issued_q = ng + 1;
        }
        const int tile = u - S.prefix[g];
        const int b = (p.q0 + S.gfirst[g]) / p.T;
        const int32_t row = (int32_t)key_row<kPaged>(p, b, (int64_t)tile * kTileKeys);
        if (kFp8) {
          const int s = k % kStg;
          ok = mbar_wait(&S.stg_empty[s], ((k / kStg) & 1) ^ 1, kErrStgEmpty);
          if (!ok) break;
          mbar_arrive_expect_tx(&S.stg_full[s], kStgBytes);
          tma_load_2d(stgbase + s * kStgBytes, &tm_k, 0, row, &S.stg_full[s]);
        } else {
          const int o = k % C::kOpN;
          ok = mbar_wait(&S.op_empty[o], ((k / C::kOpN) & 1) ^ 1, kErrOpEmpty);
          if (!ok) break;
          uint8_t* ob = opbase + o * kOpBytes;
          mbar_arrive_expect_tx(&S.op_full[o], kOpBytes);
          tma_load_2d(ob, &tm_k, 0, row, &S.op_full[o]);
          tma_load_2d(ob + kAtomBytes, &tm_k, 64, row, &S.op_full[o]);
        }
      }
      // drain: no copy into this CTA's shared memory may still be in flight at exit
      const int ring = kFp8 ? kStg : C::kOpN;
      for (int j = (k > ring ? k - ring : 0); j < k; ++j) {
        if (kFp8)
          mbar_wait(&S.stg_full[j % kStg], (uint32_t)((j / kStg) & 1), kErrStgFull);
        else
          mbar_wait(&S.op_full[j % C::kOpN], (uint32_t)((j / C::kOpN) & 1), kErrOpFull);
      }
      for (int j = (issued_q > C::kQSlots ? issued_q - C::kQSlots : 0); j < issued_q; ++j)
        mbar_wait(&S.qfull[j % C::kQSlots], (uint32_t)((j / C::kQSlots) & 1), kErrQFull);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (one lane) ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(1, kTileKeys, 64 * G);  // bf16, M = 128, N = 64 G
      const uint32_t op_s = smem_u32(opbase), q_s = smem_u32(qbase);
      int g = u0 < u1 ? find_group(S.prefix, NG, u0) : 0;
      int cur_g = -1, ng = -1, k = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u, ++k) {
        while (u >= S.prefix[g + 1]) ++g;
        if (g != cur_g) {
          if (cur_g >= 0) mma_commit(&S.qempty[ng % C::kQSlots]);  // free once its MMAs end
          ++ng;
          cur_g = g;
          ok = mbar_wait(&S.qfull[ng % C::kQSlots], (ng / C::kQSlots) & 1, kErrQFull);
          if (!ok) break;
        }
        const int o = k % C::kOpN, a = k % C::kAccN;
        ok = mbar_wait(&S.op_full[o], (uint32_t)(k / C::kOpN) & 1, kErrOpFull);
        if (!ok) break;
        ok = mbar_wait(&S.tempty[a], ((uint32_t)(k / C::kAccN) & 1) ^ 1, kErrTEmpty);
        if (!ok) break;
        tc_fence_after();
        const uint32_t ob = op_s + o * kOpBytes, qb = q_s + (ng % C::kQSlots) * C::kQSlotBytes;
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk) {  // K = 128 in steps of 16
          const uint32_t atom = kk >> 2, koff = (kk & 3) * 32;
          const uint64_t ad = smem_desc(ob + atom * kAtomBytes + koff, 16, 1024, kLayoutSw128);
          const uint64_t bd = smem_desc(qb + atom * C::kQAtomBytes + koff, 16, 1024, kLayoutSw128);
          mma_f16(tmem + (uint32_t)C::kAccCols * a, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&S.op_empty[o]);
        mma_commit(&S.tfull[a]);
      }
      mma_commit(&S.done);  // every MMA this thread issued has completed once it fires
      mbar_wait(&S.done, 0, kErrTFull);
    }
    __syncwarp();
  } else if (kFp8 && warp < 6) {
    // ------------------------------ converters (fp8) ------------------------------
    const int ct = threadIdx.x - 64;  // 0..127
    bool ok = true;
    for (int u = u0, k = 0; u < u1 && ok; ++u, ++k) {
      const int s = k % kStg, o = k % C::kOpN;
      ok = group_all_ok<3, 128>(
          mbar_wait(&S.stg_full[s], (uint32_t)(k / kStg) & 1, kErrStgFull) &&
          mbar_wait(&S.op_empty[o], ((uint32_t)(k / C::kOpN) & 1) ^ 1, kErrOpEmpty));
      if (!ok) break;
      const uint8_t* src = stgbase + s * kStgBytes;
      uint8_t* dst = opbase + o * kOpBytes;
      // a warp converts 4 rows per step: lane = (row % 4, 16-byte input chunk of 8)
      const int rsub = (ct & 31) >> 3, ic = ct & 7;
#pragma unroll 4
      for (int r0 = 4 * (ct >> 5); r0 < kTileKeys; r0 += 16) {
        const int r = r0 + rsub;
        const uint4 raw = *reinterpret_cast<const uint4*>(src + r * kDim + 16 * ic);
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t o8[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          o8[2 * j] = e4m3x2_to_bf16x2((uint16_t)(w4[j] & 0xffffu));
          o8[2 * j + 1] = e4m3x2_to_bf16x2((uint16_t)(w4[j] >> 16));
        }
        // dims 16*ic .. 16*ic+15 -> atom ic / 4, output chunks 2*(ic % 4), +1
        uint8_t* at = dst + (ic >> 2) * kAtomBytes;
        const int c8 = 2 * (ic & 3);
        *reinterpret_cast<uint4*>(at + sw128(r, c8)) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
        *reinterpret_cast<uint4*>(at + sw128(r, c8 + 1)) = make_uint4(o8[4], o8[5], o8[6], o8[7]);
      }
      fence_proxy_async_smem();  // the operand tile is read by the tensor cores
      mbar_arrive(&S.op_full[o]);
      mbar_arrive(&S.stg_empty[s]);
    }
  } else if (warp >= C::kEpiWarp0) {
    // ------------------------------ epilogue ------------------------------
    // G = 1: warps 6-9, one query; G = 4: warps 2-9, group e = members 2e, 2e+1
    constexpr int kPer = G == 1 ? 1 : 2;  // members per epilogue thread
    const int et = threadIdx.x - 32 * C::kEpiWarp0;
    const int e = G == 1 ? 0 : (warp - 2) >> 2;
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const bool hist = C::kHist && p.hist != nullptr;
    int hq = -1;
    auto flush = [&](int qq) {  // shared histogram of query qq -> global, then clear
      epi_bar<C::kEpiThreads>();
      for (int i = et; i < kBins; i += C::kEpiThreads) {
        const int v = S.hist[i];
        if (v) {
          atomicAdd(&p.hist[(size_t)qq * kBins + i], v);
          S.hist[i] = 0;
        }
      }
      epi_bar<C::kEpiThreads>();
    };
    float wr[G == 1 ? kHeads : 1];  // G = 1: the query's head weights in registers
    int cur_g = -1;
    int g = u0 < u1 ? find_group(S.prefix, NG, u0) : 0;
    bool ok = true;
    for (int u = u0, k = 0; u < u1 && ok; ++u, ++k) {
      while (u >= S.prefix[g + 1]) ++g;
      const int tile = u - S.prefix[g];
      const int f = S.gfirst[g], gs = gsize(g);
      if (g != cur_g) {
        if (G == 1) {
#pragma unroll
          for (int h = 0; h < (G == 1 ? kHeads : 1); ++h) wr[h] = p.w[(size_t)f * kHeads + h];
        } else {
          epi_bar<C::kEpiThreads>();  // every thread is done with the previous weights
          for (int i = et; i < G * kHeads; i += C::kEpiThreads) {
            const int mq = i / kHeads;
            S.wst[mq][i % kHeads] = mq < gs ? p.w[(size_t)(f + mq) * kHeads + i % kHeads] : 0.f;
          }
          epi_bar<C::kEpiThreads>();
        }
        cur_g = g;
      }
      if (hist && f != hq) {
        if (hq >= 0) flush(hq);
        hq = f;
      }
      const int s = tile * kTileKeys + 32 * quad + lane;
      const int b = (p.q0 + f) / p.T;
      // the fp8 row scale is loaded before the wait, so its latency hides behind the MMAs
      const float scale = (kFp8 && s < S.nvis[f]) ? p.key_scale[key_row<kPaged>(p, b, s)] : 1.f;
      const int a = k % C::kAccN;
      ok = group_all_ok<2, C::kEpiThreads>(
          mbar_wait(&S.tfull[a], (uint32_t)(k / C::kAccN) & 1, kErrTFull));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[kPer][kHeads];
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        tmem_ld_32x32b_x64(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)C::kAccCols * a +
                               64u * (kPer * e + j),
                           v[j]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.tempty[a]);
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int mq = kPer * e + j;  // member of the group
        if (mq >= gs) continue;
        const int q = f + mq;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh) {
          const float wv = G == 1 ? wr[hh % (G == 1 ? kHeads : 1)] : S.wst[mq][hh];
          part[hh & 3] = fmaf(wv, fmaxf(__uint_as_float(v[j][hh]), 0.f), part[hh & 3]);
        }
        float sc = (part[0] + part[1]) + (part[2] + part[3]);
        if (kFp8) sc *= scale;
        if (s < S.nvis[q]) {
          if constexpr (kB16) {  // BF16 index scores: round once, select on the rounded value
            const __nv_bfloat16 r = __float2bfloat16_rn(sc);
            p.scores16[(size_t)q * p.n_cap + s] = r;
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
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---- host: tensor maps ----
// bf16 rows of 128 values, box = 64 values (one 128-byte swizzle atom) x box_rows
bool make_map_bf16_rows(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDim * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e4m3 rows of 128 bytes, box = one 128-key tile, no swizzle (the converters read it)
bool make_map_fp8_rows(CUtensorMap* m, const void* ptr, uint64_t rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDim};
  cuuint32_t box[2] = {(cuuint32_t)kDim, (cuuint32_t)kTileKeys};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kFp8, int G>
size_t smem_bytes() {
  using C = Cfg<kFp8, G>;
  return 1024 + (size_t)C::kOpN * kOpBytes + (size_t)C::kQSlots * C::kQSlotBytes +
         (kFp8 ? (size_t)kStg * kStgBytes : 0) + sizeof(Smem<C::kHist>);
}

template <bool kFp8, int G, bool kB16, bool kPaged>
cudaError_t launch_variant(const CUtensorMap& mk, const CUtensorMap& mq, const Bf16IdxParams& p,
                           int grid, cudaStream_t st) {
  const size_t smem = smem_bytes<kFp8, G>();
  cudaError_t e = cudaFuncSetAttribute(k_index_bf16_tc<kFp8, G, kB16, kPaged>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch(true, k_index_bf16_tc<kFp8, G, kB16, kPaged>, dim3(grid), dim3(kThreads), smem,
                st, mk, mq, p);
}

template <bool kB16, bool kPaged>
cudaError_t launch_one(bool fp8, bool grp, const CUtensorMap& mk, const CUtensorMap& mq,
                       const Bf16IdxParams& p, int grid, cudaStream_t st) {
  return fp8   ? launch_variant<true, 1, kB16, kPaged>(mk, mq, p, grid, st)
         : grp ? launch_variant<false, 4, kB16, kPaged>(mk, mq, p, grid, st)
               : launch_variant<false, 1, kB16, kPaged>(mk, mq, p, grid, st);
}

}  // namespace

bool index_bf16_tc_supported(const IndexArgs& a) {
  const bool rows_ok = a.page_table == nullptr
                           ? (int64_t)a.B * a.n_cap < (1ll << 31)
                           : a.page_rows % kTileKeys == 0 &&
                                 (int64_t)a.n_pages * a.page_rows < (1ll << 31);
  return (a.kdt == CSA_FP8_E4M3_ROWSCALE || a.kdt == CSA_BF16) && a.n_idx_heads == kHeads &&
         a.d_idx == kDim && a.n_cap % kTileKeys == 0 && rows_ok;
}

cudaError_t launch_index_bf16_tc(const IndexArgs& a, cudaStream_t st) {
  const int Qall = a.B * a.T;
  const bool fp8 = a.kdt == CSA_FP8_E4M3_ROWSCALE;
  // four queries of a request per MMA (N = 256) when several share the keys and no per-query
  // histogram is wanted (bf16 keys, prefill); otherwise one
  const bool grouped = !fp8 && a.hist == nullptr && a.T >= 4;
  const bool paged = a.page_table != nullptr;
  const uint64_t key_rows = paged ? (uint64_t)a.n_pages * a.page_rows : (uint64_t)a.B * a.n_cap;
  CUtensorMap mk;
  const bool good = fp8 ? make_map_fp8_rows(&mk, a.KI, key_rows)
                        : make_map_bf16_rows(&mk, a.KI, key_rows, kTileKeys);
  if (!good) return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  timing_before(st);
  // queries in launches of at most kMaxQueries (each launch walks its groups' tiles)
  for (int q0 = 0; q0 < Qall && e == cudaSuccess; q0 += kMaxQueries) {
    const int Q = Qall - q0 < kMaxQueries ? Qall - q0 : kMaxQueries;
    // a batch of fewer than four queries (a tail) has fewer q rows than a group's box
    const bool grp = grouped && Q >= 4;
    CUtensorMap mq;
    const auto* qI = static_cast<const __nv_bfloat16*>(a.qI) + (size_t)q0 * kHeads * kDim;
    if (!make_map_bf16_rows(&mq, qI, (uint64_t)Q * kHeads, grp ? 4 * kHeads : kHeads)) {
      e = cudaErrorInvalidValue;
      break;
    }
    const bool b16 = a.scores16 != nullptr;
    Bf16IdxParams p{Q, a.T, a.m, q0, a.n_cap, a.q_pos + q0, a.w + (size_t)q0 * kHeads,
                    fp8 ? static_cast<const float*>(a.KI_scale) : nullptr,
                    b16 ? nullptr : a.scores + (size_t)q0 * a.n_cap,
                    a.hist ? a.hist + (size_t)q0 * kBins : nullptr,
                    b16 ? static_cast<__nv_bfloat16*>(a.scores16) + (size_t)q0 * a.n_cap : nullptr,
                    a.page_table, a.page_rows, a.max_pages, a.n_pages};
    const int64_t tiles_max = (int64_t)Q * (a.n_cap / kTileKeys);
    const int grid = (int)(tiles_max < device_sm_count() ? (tiles_max > 0 ? tiles_max : 1) : device_sm_count());
    e = paged ? (b16 ? launch_one<true, true>(fp8, grp, mk, mq, p, grid, st)
                     : launch_one<false, true>(fp8, grp, mk, mq, p, grid, st))
              : (b16 ? launch_one<true, false>(fp8, grp, mk, mq, p, grid, st)
                     : launch_one<false, false>(fp8, grp, mk, mq, p, grid, st));
  }
  timing_after(st);
  return e;
}

cudaError_t index_bf16_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, tc::g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));
}

}  // namespace csa
