// Stage 4 on tensor cores: shared-KV MQA (sparse CSA rows or dense HCA rows) plus the
// sliding window, with query RMSNorm / RoPE, sink and output un-rotation.
//
// 【论文解读】DeepSeek-V4 一(三)1(3) / 2(2): every KV row is key and value for all heads;
// 3(1) RMSNorm of each query head; 3(2) RoPE(t) on the last r dims of q, RoPE(-t) on the
// output; 3(3) window rows attended with the compressed rows; 3(4) exp(z'_h) added to the
// softmax denominator.
//
// Work: a stream is (query, group of 64 heads); its KV row list (selected or visible
// entries, then the window) is cut into chunks of 128 rows (one buffer) or, when a CTA walks
// several, 64 rows (two buffers: the next chunk's rows arrive during this one's softmax),
// and the chunks of a stream are split over `nsplit` CTAs. Per chunk of R rows, with bf16
// operands in 128B-swizzled shared memory and fp32 accumulators in TMEM:
//   S[64 heads x R rows] = q_hat . K_chunk^T            (A = q_hat, M = 64; B = KV tile)
//   P = exp(S * scale - m_h) in bf16                    (softmax: thread = head, its R
//                                                        row values in registers)
//   O^T[4 x 128 dims x 64 heads] += V_chunk^T . P^T     (A = the same KV tile read MN-major,
//                                                        B = P, K-major)
// so the gathered tile is read from shared memory by both products and never transposed,
// and every per-head reduction (max, sum) stays inside one thread.
// The running max m_h is only raised when a chunk's max exceeds it by more than 8 (then
// O^T and l are rescaled); exp(s - m) <= e^8 otherwise, exactly as correct.
// One split: the CTA finalises (sink, RoPE(-t), bf16). Several: it writes (m, l, O)
// partials and k_mqa_combine merges them in a fixed order (deterministic).
//
// Mixed-precision KV rows (一(三)4 item 1: RoPE dims in BF16, the rest in FP8; kMixed):
// a cache row is c + r bytes, the e4m3 codes of its first c - r values (one fp32 scale per
// row) then its last r values as bf16. The gather widens code * scale to bf16 into the
// same swizzled tile (one rounding) and copies the bf16 values as they are, so the tensor
// core work is unchanged and each selected row moves 580 bytes instead of 1024. Window rows
// stay bf16.
//
// Paged cache (kPaged; 二、基础设施 (六) 推理框架): the classical cache is a pool of pages and
// a request's entry e is row e % page_rows of page page_table[b, e / page_rows]; only the
// gather's address changes. A page id outside the pool masks the row and records an error.
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "host_util.cuh"
#include "internal.h"
#include "tc.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kC = 512;          // head dim
constexpr int kHg = 64;          // heads per CTA (MMA N)
constexpr int kThreads = 160;    // warps 0-3: loads + softmax + epilogue; warp 4: MMA
constexpr int kAtoms = kC / 64;  // 64-element (128 B) swizzle atoms along a row
constexpr float kLazy = 8.f;     // rescale threshold (natural-log units)
constexpr int kMaxPairs = 256;   // RoPE pairs (r / 2)

// Shared memory (offsets from a 1024-aligned base) for chunks of kR KV rows: kR = 128 with
// one KV buffer, or kR = 64 with two (the next chunk's rows arrive while this one's products
// and softmax run). 208 KB either way; the KV area also stages the 64 raw query rows (64 KB)
// before q_hat is built.
template <int kR>
struct Lay {
  static constexpr int kBuf = kR == 64 ? 2 : 1;
  static constexpr int kSlotKV = kAtoms * kR * 128;                   // [atom][row][128 B]
  static constexpr int kOffKV = 0;
  static constexpr int kOffQ = kOffKV + kBuf * kSlotKV;              // [atom][head][128 B]
  static constexpr int kSlotP = kR * 128;                             // [row / 64][head][128 B]
  static constexpr int kOffP = kOffQ + kAtoms * kHg * 128;
  static constexpr int kOffEnd = kOffP + kBuf * kSlotP;
};

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // S: 128 columns (M = 64 layout)
constexpr uint32_t kColO = 256;   // O^T slice s: 256 + 64 s

enum { kErrKvFull = 201, kErrSFull = 202, kErrPFull = 203, kErrKvFree = 204, kErrPageId = 205 };

template <bool kMixed, int kR>
struct SmemT {
  static constexpr int kBuf = Lay<kR>::kBuf;
  uint64_t kv_full[kBuf], s_full[kBuf], p_full[kBuf], kv_free[kBuf], done;
  uint32_t tmem_slot;
  uint32_t vmask[kBuf][kR / 32];  // valid rows of a buffered chunk (bit j of word w: row 32w + j)
  float m_used[kHg], l_sum[kHg], alpha[kHg], fin[kHg];
  float cs[kMaxPairs], sn[kMaxPairs];  // RoPE table for pairs of the last r dims
  float wq[kC];                         // query RMSNorm weights
  // per buffer: source rows of the chunk being gathered (nullptr: masked) and, for mixed
  // rows, the row's FP8 scale (bf16 rows: -1); one set per buffer, since the next chunk's
  // rows are resolved while other warps may still be copying this one's
  const __nv_bfloat16* src[kBuf][kR];
  float rscale[kBuf][kMixed ? kR : 1];
};

struct MqaTcParams {
  MqaArgs a;
  int G;       // head groups (H / 64)
  int nsplit;  // CTAs per stream
  float* part; // partials [stream][split][64 * (kC + 2)] or nullptr
  int tma_kv, tma_win;  // tensor maps usable for chunks of contiguous cache / window rows
  double inv_freq[kMaxPairs];  // RoPE pair frequencies base^(-2p/r), formed once on the host
};

__device__ __forceinline__ void bar_softmax() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// AND of `ok` over the 128 softmax threads (keeps them in lockstep when a wait gives up).
__device__ __forceinline__ bool all_ok_softmax(bool ok) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(res)
      : "r"((uint32_t)ok)
      : "memory");
  return res != 0;
}

// OR of `p` over the 128 softmax threads.
__device__ __forceinline__ bool any_softmax(bool p) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(res)
      : "r"((uint32_t)p)
      : "memory");
  return res != 0;
}

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Row list of a query: [selected (k) or visible (n_vis) entries][window tokens].
struct RowList {
  int64_t t, n_vis, n_sel, lo, n_w, L;
};

__device__ __forceinline__ RowList row_list(const MqaArgs& a, int bt) {
  RowList r;
  r.t = a.q_pos[bt];
  r.n_vis = r.t < 0 ? 0 : (r.t / a.m < a.n_cap ? r.t / a.m : a.n_cap);
  r.n_sel = a.k > 0 ? a.k : r.n_vis;
  r.lo = (r.t - a.n_win + 1) > 0 ? (r.t - a.n_win + 1) : 0;
  r.n_w = (a.n_win > 0 && r.t >= 0) ? r.t - r.lo + 1 : 0;
  r.L = r.n_sel + r.n_w;
  return r;
}

// Source row of list entry j (nullptr: masked).
__device__ __forceinline__ const __nv_bfloat16* row_src(const MqaArgs& a, int bt, int b,
                                                        const RowList& rl, int64_t j) {
  if (j < rl.n_sel) {
    int64_t e = j;
    if (a.k > 0) e = a.idx[(size_t)bt * a.k + j];
    else if (e >= rl.n_vis) return nullptr;
    if (e < 0 || e >= a.n_cap) return nullptr;
    return static_cast<const __nv_bfloat16*>(a.kv) + ((size_t)b * a.n_cap + e) * kC;
  }
  if (j < rl.L) {
    const int64_t rr = rl.lo + (j - rl.n_sel) - a.win_pos0[b];
    if (rr < 0 || rr >= a.l_raw) return nullptr;
    return static_cast<const __nv_bfloat16*>(a.win) + ((size_t)b * a.l_raw + rr) * kC;
  }
  return nullptr;
}

// Source of list entry j for the mixed-precision and / or paged variants: a cache row (bf16,
// or c + r mixed bytes with its scale in *scale) found through the page table when kPaged,
// or a bf16 window row (*scale = -1); nullptr when masked. pg_hint >= -1: the entry's page
// id, read earlier.
template <bool kMixed, bool kPaged>
__device__ __forceinline__ const void* row_src_ext(const MqaArgs& a, int bt, int b,
                                                   const RowList& rl, int64_t j, float* scale,
                                                   int32_t pg_hint = -2) {
  *scale = -1.f;
  if (j < rl.n_sel) {
    int64_t e = j;
    if (a.k > 0) e = a.idx[(size_t)bt * a.k + j];
    else if (e >= rl.n_vis) return nullptr;
    if (e < 0 || e >= a.n_cap) return nullptr;
    size_t row = (size_t)b * a.n_cap + e;
    if constexpr (kPaged) {
      const int32_t pg =
          pg_hint >= -1 ? pg_hint : a.page_table[(size_t)b * a.max_pages + e / a.page_rows];
      if (pg < 0 || pg >= a.n_pages) {
        set_error(kErrPageId);
        return nullptr;
      }
      row = (size_t)pg * a.page_rows + (size_t)(e % a.page_rows);
    }
    if constexpr (kMixed) {
      *scale = a.kv_scale[row];
      return static_cast<const uint8_t*>(a.kv) + row * (size_t)(kC + a.rope_dims);
    } else {
      return static_cast<const __nv_bfloat16*>(a.kv) + row * kC;
    }
  }
  if (j < rl.L) {
    const int64_t p = rl.lo + (j - rl.n_sel);  // the window token's position
    // win_pos0 == nullptr: the state cache's window ring (position p in row p mod l_raw)
    const int64_t rr = a.win_pos0 != nullptr ? p - a.win_pos0[b] : p % a.l_raw;
    if (rr < 0 || rr >= a.l_raw) return nullptr;
    return static_cast<const __nv_bfloat16*>(a.win) + ((size_t)b * a.l_raw + rr) * kC;
  }
  return nullptr;
}

// two e4m3 codes (low byte first) times `scale`, rounded to bf16x2
__device__ __forceinline__ uint32_t e4m3x2_scaled_bf16x2(uint32_t v, float scale) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)v));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  const __nv_bfloat162 r = __floats2bfloat162_rn(f.x * scale, f.y * scale);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// 32 lanes x 16 columns of 32-bit: thread i of the warp gets lane (quadrant*32 + i).
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// 16 TMEM lanes x 64 columns of 32-bit, two threads per lane: thread t of the warp gets lane
// (quadrant base + t / 4 + 8 (t % 2)) and, in register i, column 2 i + (t / 2) % 2 (the
// layout checked on the device by writing known values through the 32x32b shape).
__device__ __forceinline__ void tmem_ld_16x64b_x32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x64b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
      " [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Reduce 16 per-thread values over the warp's 32 threads: on return lanes 2j and 2j+1 both
// hold the reduction of value j (4 halving exchanges, then one pairwise exchange).
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16]) {
  const int lane = threadIdx.x & 31;
  float a8[8], a4[4], a2[2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    const float got = __shfl_xor_sync(0xffffffffu, hi ? v[i] : v[8 + i], 16);
    const float keep = hi ? v[8 + i] : v[i];
    a8[i] = kMax ? fmaxf(keep, got) : keep + got;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    const float got = __shfl_xor_sync(0xffffffffu, hi ? a8[i] : a8[4 + i], 8);
    const float keep = hi ? a8[4 + i] : a8[i];
    a4[i] = kMax ? fmaxf(keep, got) : keep + got;
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    const float got = __shfl_xor_sync(0xffffffffu, hi ? a4[i] : a4[2 + i], 4);
    const float keep = hi ? a4[2 + i] : a4[i];
    a2[i] = kMax ? fmaxf(keep, got) : keep + got;
  }
  const bool hi = lane & 2;
  const float got = __shfl_xor_sync(0xffffffffu, hi ? a2[0] : a2[1], 2);
  float r = hi ? a2[1] : a2[0];
  r = kMax ? fmaxf(r, got) : r + got;
  const float other = __shfl_xor_sync(0xffffffffu, r, 1);
  return kMax ? fmaxf(r, other) : r + other;
}

template <bool kMixed, bool kPaged, int kRows>
__global__ void __launch_bounds__(kThreads, 1)
    k_mqa_tc(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_win,
             MqaTcParams P) {
  using Smem = SmemT<kMixed, kRows>;
  using L = Lay<kRows>;
  constexpr int kBuf = L::kBuf, kOffKV = L::kOffKV, kOffQ = L::kOffQ, kOffP = L::kOffP,
                kOffEnd = L::kOffEnd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  Smem& S = *reinterpret_cast<Smem*>(base + kOffEnd);
  const MqaArgs& a = P.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int stream = blockIdx.x / P.nsplit, split = blockIdx.x % P.nsplit;
  const int bt = stream / P.G, g = stream % P.G;
  const int b = bt / a.T;
  const int h0 = g * kHg;
  const RowList rl = row_list(a, bt);
  const int nchunks = (int)((rl.L + kRows - 1) / kRows);
  const int c0 = (int)(((int64_t)nchunks * split) / P.nsplit);
  const int c1 = (int)(((int64_t)nchunks * (split + 1)) / P.nsplit);
  const int r = a.rope_dims, r0 = kC - r;
  // Without a programmatic launch every input is complete when the kernel starts, so with
  // two KV buffers the first chunk's rows are requested before q_hat is built (the raw
  // query rows are staged in the second buffer).
  const bool early = kBuf == 2 && !a.chained && c0 < c1;
  uint8_t* const q_stage = base + kOffKV + (kBuf == 2 ? L::kSlotKV : 0);

  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < kBuf; ++i) {
        mbar_init(&S.kv_full[i], 129);  // the 128 loading threads + the TMA issue or its stand-in
        mbar_init(&S.s_full[i], 1);
        mbar_init(&S.p_full[i], 128);
        mbar_init(&S.kv_free[i], 1);
      }
      mbar_init(&S.done, 1);
      fence_barrier_init();
    }
    tmem_alloc(&S.tmem_slot, kTmemCols);
  } else {
    if (a.qhat != nullptr) {
      // q_hat was prepared by an earlier kernel: copy it straight into the B-operand tile
      const uint4* qg = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.qhat) +
                                                       ((size_t)bt * a.H + h0) * kC);
      const uint32_t qt = smem_u32(base + kOffQ);
#pragma unroll 4
      for (int i = tid; i < kHg * kC / 8; i += 128) {
        const int h = i >> 6, d0 = 8 * (i & 63);
        cp_async16(qt + (d0 >> 6) * (kHg * 128) + sw128(h, (d0 & 63) >> 3), qg + i, true);
      }
    } else {
      // the group's 64 raw query rows (64 KB, contiguous) into a KV buffer that no gather
      // overwrites before q_hat is built; one pass, one latency
      const uint32_t stage = smem_u32(q_stage);
      const uint4* qg = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                       ((size_t)bt * a.H + h0) * kC);
#pragma unroll 4
      for (int i = tid; i < kHg * kC / 8; i += 128) cp_async16(stage + 16 * i, qg + i, true);
    }
    // RoPE table, norm weights and running stats while the copies are in flight
    for (int p = tid; p < r / 2; p += 128)
      rope_angle_cs((double)rl.t, P.inv_freq[p], &S.cs[p], &S.sn[p]);
    for (int d = tid; d < kC; d += 128)
      S.wq[d] = a.q_rms_w ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q_rms_w)[d]) : 1.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_slot;

  if (warp < 4) {
    // A chunk's rows are gathered in two steps: the issue (rows resolved, copies or TMA boxes
    // started; returns whether TMA fills the slot) and the finish (cp.async copies: wait for
    // this thread's, make them visible to the tensor cores; then arrive). With two buffers the
    // next chunk is issued before this one's softmax and finished after it.
    // dense paged lists: the page ids of the next chunk's rows are read one chunk ahead, so
    // that resolving a chunk's rows waits on no page-table load
    int pf_j = -1;
    int32_t pf_pg = -2;
    auto gather_issue = [&](int j, int slot) -> bool {
      // ---- rows of chunk j into KV slot `slot`: thread r resolves row r, then warp w copies
      //      rows w, w+4, ... with lane = 16-byte chunk (coalesced 512 B per instruction) ----
      const uint32_t kv_base = smem_u32(base + kOffKV + slot * L::kSlotKV);
      uint8_t* const kv_ptr = base + kOffKV + slot * L::kSlotKV;
      const __nv_bfloat16* my_src = nullptr;
      if (tid < kRows) {
        if constexpr (kMixed || kPaged) {
          float sc;
          my_src = static_cast<const __nv_bfloat16*>(row_src_ext<kMixed, kPaged>(
              a, bt, b, rl, (int64_t)j * kRows + tid, &sc, pf_j == j ? pf_pg : -2));
          if constexpr (kMixed) S.rscale[slot][tid] = sc;
          if constexpr (kPaged) {
            const int64_t e1 = (int64_t)(j + 1) * kRows + tid;
            pf_pg = -2;
            if (a.k == 0 && j + 1 < c1 && e1 < rl.n_vis && e1 < a.n_cap)
              pf_pg = a.page_table[(size_t)b * a.max_pages + e1 / a.page_rows];
            pf_j = j + 1;
          }
        } else {
          my_src = row_src(a, bt, b, rl, (int64_t)j * kRows + tid);
        }
        S.src[slot][tid] = my_src;
      }
      const uint32_t vb = __ballot_sync(0xffffffffu, my_src != nullptr);
      if (lane == 0 && warp < kRows / 32) S.vmask[slot][warp] = vb;
      // a chunk of 128 contiguous rows (dense entries, or window rows) comes by TMA: eight
      // 128B-swizzled boxes issued by one thread instead of 64 cp.async per thread
      const int64_t r0 = (int64_t)j * kRows;
      const CUtensorMap* tmap = nullptr;
      int32_t trow = 0;
      if (P.tma_kv && a.k == 0 && r0 + kRows <= rl.n_vis) {
        tmap = &tm_kv;
        trow = (int32_t)((int64_t)b * a.n_cap + r0);
      } else if (P.tma_win && r0 >= rl.n_sel && r0 + kRows <= rl.L) {
        const int64_t rr0 = rl.lo + (r0 - rl.n_sel) - a.win_pos0[b];
        if (rr0 >= 0 && rr0 + kRows <= a.l_raw) {
          tmap = &tm_win;
          trow = (int32_t)((int64_t)b * a.l_raw + rr0);
        }
      }
      bar_softmax();
      if (tmap != nullptr) {
        if (tid == 0) {
          mbar_arrive_expect_tx(&S.kv_full[slot], kRows * kC * 2);
#pragma unroll
          for (int atom = 0; atom < kAtoms; ++atom)
            tma_load_2d(kv_ptr + atom * (kRows * 128), tmap, 64 * atom, trow, &S.kv_full[slot]);
        }
        return true;
      } else {
        if constexpr (kMixed) {
          // a warp takes rows w, w+4, ...: a mixed row's lanes 0..27 widen 16 codes each
          // (dims 16*lane ..: atom lane / 4, chunks 2*(lane % 4) and +1), lanes 28..31 copy
          // two 16-byte chunks of its bf16 RoPE values (dims 448 + 8*q: atom 7, chunk q);
          // a bf16 window row (scale -1) or a masked row is copied as in the bf16 path. Four
          // rows at a time: their code loads are all issued before any is widened, so the
          // warp waits for one round trip per four rows.
          const int r = a.rope_dims, nope = kC - r;  // nope = 448 (c = 512, r = 64)
#pragma unroll 1
          for (int rb = warp; rb < kRows; rb += 16) {  // rows rb, rb + 4, rb + 8, rb + 12
            uint4 raw[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const __nv_bfloat16* src = S.src[slot][rb + 4 * q];
              raw[q] = make_uint4(0u, 0u, 0u, 0u);
              if (src != nullptr && S.rscale[slot][rb + 4 * q] >= 0.f && lane < nope / 16)
                raw[q] = __ldg(reinterpret_cast<const uint4*>(src) + lane);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int rr = rb + 4 * q;
              const __nv_bfloat16* src = S.src[slot][rr];
              const float sc = S.rscale[slot][rr];
              if (src == nullptr || sc < 0.f) {
#pragma unroll
                for (int hseg = 0; hseg < 2; ++hseg) {
                  const int gch = lane + 32 * hseg;
                  const int atom = gch >> 3, c = gch & 7;
                  const uint32_t dst = kv_base + atom * (kRows * 128) + sw128(rr, c);
                  cp_async16(dst, src ? src + 8 * gch : static_cast<const __nv_bfloat16*>(a.kv),
                             src != nullptr);
                }
              } else {
                const uint8_t* row = reinterpret_cast<const uint8_t*>(src);
                if (lane < nope / 16) {
                  const uint32_t w4[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
                  uint32_t o8[8];
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    o8[2 * e] = e4m3x2_scaled_bf16x2(w4[e] & 0xffffu, sc);
                    o8[2 * e + 1] = e4m3x2_scaled_bf16x2(w4[e] >> 16, sc);
                  }
                  uint8_t* at = kv_ptr + (lane >> 2) * (kRows * 128);
                  const int c8 = 2 * (lane & 3);
                  *reinterpret_cast<uint4*>(at + sw128(rr, c8)) =
                      make_uint4(o8[0], o8[1], o8[2], o8[3]);
                  *reinterpret_cast<uint4*>(at + sw128(rr, c8 + 1)) =
                      make_uint4(o8[4], o8[5], o8[6], o8[7]);
                } else {
                  const int q0 = 2 * (lane - nope / 16);  // RoPE chunks q0, q0 + 1 of r / 8
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const int qq = q0 + h;
                    if (qq < r / 8) {
                      const int d = nope + 8 * qq;
                      const uint32_t dst =
                          kv_base + (d >> 6) * (kRows * 128) + sw128(rr, (d & 63) >> 3);
                      cp_async16(dst, row + nope + 16 * qq, true);
                    }
                  }
                }
              }
            }
          }
        } else {
#pragma unroll 4
          for (int rr = warp; rr < kRows; rr += 4) {
            const __nv_bfloat16* src = S.src[slot][rr];
#pragma unroll
            for (int hseg = 0; hseg < 2; ++hseg) {
              const int gch = lane + 32 * hseg;  // 16-byte chunk of the 1 KB row
              const int atom = gch >> 3, c = gch & 7;
              const uint32_t dst = kv_base + atom * (kRows * 128) + sw128(rr, c);
              cp_async16(dst, src ? src + 8 * gch : static_cast<const __nv_bfloat16*>(a.kv),
                         src != nullptr);
            }
          }
        }
        return false;
      }
    };
    auto gather_finish = [&](int slot, bool tma) {
      if (!tma) {
        cp_async_wait_all();
        fence_proxy_async_smem();
        if (tid == 0) mbar_arrive(&S.kv_full[slot]);  // stands in for the TMA issue
      }
      mbar_arrive(&S.kv_full[slot]);
    };
    int pend = -1;  // slot of a gather issued and not yet finished
    bool pend_tma = false;
    if constexpr (kBuf == 2) {
      if (early) {
        pend_tma = gather_issue(c0, 0);
        pend = 0;
      }
    }
    if (a.qhat != nullptr) {
      cp_async_wait_all();
      fence_proxy_async_smem();  // the tile is read by the tensor cores
    } else {
      // ---- q_hat = RoPE_t(RMSNorm(q)) in bf16: two threads per head, 256 dims each. Thread
      //      t reads its 32 chunks of 8 dims starting at chunk t % 32, so that a warp's reads
      //      of one step spread over all banks. ----
      uint8_t* qs = base + kOffQ;
      const int qh = tid >> 1, qhalf = tid & 1;
      const uint4* qrow = reinterpret_cast<const uint4*>(q_stage + qh * (kC * 2)) + 32 * qhalf;
      cp_async_wait_all();
      bar_softmax();
      float ss0 = 0.f, ss1 = 0.f;
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        const uint4 raw = qrow[(i + lane) & 31];
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float lo = __uint_as_float(w4[k] << 16), hi = __uint_as_float(w4[k] & 0xffff0000u);
          ss0 = fmaf(lo, lo, ss0);
          ss1 = fmaf(hi, hi, ss1);
        }
      }
      float ss = ss0 + ss1;
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      const float rstd = rsqrtf(ss / (float)kC + a.eps);
#pragma unroll 4
      for (int i = 0; i < 32; ++i) {
        const int c = (i + lane) & 31;
        const uint4 raw = qrow[c];
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
        const int d0 = 256 * qhalf + 8 * c;
        float y[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          y[2 * k] = __uint_as_float(w4[k] << 16) * rstd * S.wq[d0 + 2 * k];
          y[2 * k + 1] = __uint_as_float(w4[k] & 0xffff0000u) * rstd * S.wq[d0 + 2 * k + 1];
        }
        if (d0 >= r0) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int p = (d0 + 2 * k - r0) >> 1;
            const float cs = S.cs[p], sn = S.sn[p], u = y[2 * k], v = y[2 * k + 1];
            y[2 * k] = u * cs - v * sn;
            y[2 * k + 1] = u * sn + v * cs;
          }
        }
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ow[k] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * k])) |
                  ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * k + 1])) << 16);
        const int atom = d0 >> 6, chunk = (d0 & 63) >> 3;
        *reinterpret_cast<uint4*>(qs + atom * (kHg * 128) + sw128(qh, chunk)) = o;
      }
      // the tile is read by the tensor cores, also when a chunk's rows come by TMA (whose
      // arrival carries no fence of these stores)
      fence_proxy_async_smem();
    }

    // the selected rows, the partials and the output belong to the previous kernels
    pdl_wait();
    pdl_trigger();
    bool ok = true;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    // the M = 64 accumulator puts head 16w + i in TMEM lane 32w + i (i < 16); threads t and
    // t ^ 2 of warp w share head 16w + t / 4 + 8 (t % 2), each holding every other row of a
    // chunk (rows 2i + par)
    const int par = (lane >> 1) & 1;
    const int hh = 16 * warp + (lane >> 2) + 8 * (lane & 1);
    float mu_h = -INFINITY, l_h = 0.f;  // running max used and running sum of this head
    if (c0 < c1 && pend < 0) {
      pend_tma = gather_issue(c0, 0);
      pend = 0;
    }
#pragma unroll 1
    for (int j = c0; j < c1 && ok; ++j) {
      const uint32_t it = (uint32_t)(j - c0);
      const int slot = (int)(it % kBuf);
      const uint32_t ph = (it / kBuf) & 1;
      if constexpr (kBuf == 1) {
        if (j > c0) {  // the previous chunk's O^T products are done: the buffer is free
          ok = all_ok_softmax(mbar_wait(&S.kv_free[0], (it - 1) & 1, kErrKvFree));
          if (!ok) break;
          pend_tma = gather_issue(j, 0);
          pend = 0;
        }
        gather_finish(0, pend_tma);
        pend = -1;
      } else {
        if (j == c0) {
          gather_finish(0, pend_tma);
          pend = -1;
        } else {  // O(j-1) done: its buffer may take chunk j+1, and O^T may be rescaled
          ok = all_ok_softmax(mbar_wait(&S.kv_free[(it + 1) & 1], ((it - 1) >> 1) & 1, kErrKvFree));
          if (!ok) break;
        }
        if (j + 1 < c1) {
          pend_tma = gather_issue(j + 1, (int)((it + 1) & 1));
          pend = (int)((it + 1) & 1);
        }
      }

      // ---- softmax: the two threads of head hh hold its rows 2i + par (i < R / 2); each
      //      reduction is the thread's own values and one exchange with its partner ----
      ok = all_ok_softmax(mbar_wait(&S.s_full[slot], ph, kErrSFull));
      if (!ok) break;
      tc_fence_after();
      constexpr int kV = kRows / 2;  // values per thread
      uint32_t sv[kV];
#pragma unroll
      for (int h = 0; h < kRows / 64; ++h)
        tmem_ld_16x64b_x32(lane_base + kColS + (kBuf == 2 ? 64 * slot : 0) + 64 * h, sv + 32 * h);
      tmem_ld_wait();
      uint32_t vm[kRows / 32];
#pragma unroll
      for (int i = 0; i < kRows / 32; ++i) vm[i] = S.vmask[slot][i];
      // scaled logits in place (masked rows -> -inf); eight partial maxima keep the
      // dependency chains short (max is exact in any order)
      float cmx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cmx[i] = -INFINITY;
#pragma unroll
      for (int i = 0; i < kV; ++i) {
        const int rr = 2 * i + par;
        const float x =
            ((vm[rr >> 5] >> (rr & 31)) & 1u) ? __uint_as_float(sv[i]) * a.scale : -INFINITY;
        sv[i] = __float_as_uint(x);
        cmx[i & 7] = fmaxf(cmx[i & 7], x);
      }
      float cm = fmaxf(fmaxf(fmaxf(cmx[0], cmx[1]), fmaxf(cmx[2], cmx[3])),
                       fmaxf(fmaxf(cmx[4], cmx[5]), fmaxf(cmx[6], cmx[7])));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
      float al = 1.f;
      if (cm > mu_h + kLazy || (mu_h == -INFINITY && cm != -INFINITY)) {
        al = (mu_h == -INFINITY) ? 0.f : expf(mu_h - cm);
        mu_h = cm;
      }
      l_h *= al;
      if (par == 0) S.alpha[hh] = al;
      if (any_softmax(al != 1.f && j > c0)) {
        // rare: scale O^T columns by alpha (the previous O^T MMAs are done)
#pragma unroll 1
        for (int cgrp = 0; cgrp < 16; ++cgrp) {  // 4 slices x 4 groups of 16 heads
          uint32_t o[16];
          const uint32_t ta = lane_base + kColO + 16 * cgrp;
          tmem_ld_x16(ta, o);
          tmem_ld_wait();
          const int hb = 16 * (cgrp & 3);
#pragma unroll
          for (int h = 0; h < 16; ++h)
            o[h] = __float_as_uint(__uint_as_float(o[h]) * S.alpha[hb + h]);
          tmem_st_x16(ta, o);
        }
        tmem_st_wait();
      }
      // P row of this head (bf16) into the K-major B tile [row / 64][head][128 B]. Per 16
      // rows the even thread writes rows 0-7 and the odd thread rows 8-15: each hands its
      // partner the four values the partner's 16-byte chunk needs.
      {
        uint8_t* pt = base + kOffP + slot * L::kSlotP;
        float lc[4] = {0.f, 0.f, 0.f, 0.f};  // partial sums (sum what the MMA multiplies)
        const float mref = mu_h == -INFINITY ? 0.f : mu_h;  // no valid row yet: every p is 0
#pragma unroll
        for (int g = 0; g < kRows / 16; ++g) {
          uint32_t bb[8];  // bf16 bits of rows 16g + 2m + par
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const __nv_bfloat16 bv = __float2bfloat16_rn(__expf(__uint_as_float(sv[8 * g + m]) - mref));
            lc[m & 3] += __bfloat162float(bv);
            bb[m] = (uint32_t)__bfloat16_as_ushort(bv);
          }
          const uint32_t s0 = par ? (bb[0] | (bb[1] << 16)) : (bb[4] | (bb[5] << 16));
          const uint32_t s1 = par ? (bb[2] | (bb[3] << 16)) : (bb[6] | (bb[7] << 16));
          const uint32_t r0 = __shfl_xor_sync(0xffffffffu, s0, 2);
          const uint32_t r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
          const uint32_t pk[4] = {r0 & 0xffffu, r0 >> 16, r1 & 0xffffu, r1 >> 16};
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t own = par ? bb[4 + k] : bb[k];
            w[k] = par ? (pk[k] | (own << 16)) : (own | (pk[k] << 16));
          }
          const int c8 = 2 * g + par;  // 16-byte chunk: rows 8 c8 .. 8 c8 + 7
          *reinterpret_cast<uint4*>(pt + (c8 >> 3) * (kHg * 128) + sw128(hh, c8 & 7)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_h += (lc[0] + lc[1]) + (lc[2] + lc[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&S.p_full[slot]);
      if constexpr (kBuf == 2) {
        if (pend >= 0) {  // the next chunk's rows: in flight during this softmax, landed now
          gather_finish(pend, pend_tma);
          pend = -1;
        }
      }
    }
    if (pend >= 0) cp_async_wait_all();  // a wait gave up: no copy of this thread in flight
    l_h += __shfl_xor_sync(0xffffffffu, l_h, 2);  // the two halves of the head's sum
    if (par == 0) {
      S.m_used[hh] = mu_h;
      S.l_sum[hh] = l_h;
    }
    // ---- epilogue: wait for the last O^T, then finalise or write the partial ----
    if (ok && c1 > c0) {
      const uint32_t last = (uint32_t)(c1 - c0 - 1);
      ok = all_ok_softmax(mbar_wait(&S.kv_free[last % kBuf], (last / kBuf) & 1, kErrKvFree));
    }
    bar_softmax();
    const bool single = P.nsplit == 1;
    if (tid < kHg) {
      const float m = S.m_used[tid], l = S.l_sum[tid];
      if (single) {
        const float zs = a.sink ? a.sink[h0 + tid] : -INFINITY;
        float f = 0.f;
        if (l > 0.f) {
          const float M = fmaxf(m, zs);
          f = expf(m - M) / (l * expf(m - M) + (zs == -INFINITY ? 0.f : expf(zs - M)));
        }
        S.fin[tid] = f;
      } else {
        float* pp = P.part + ((size_t)stream * P.nsplit + split) * (kHg * (kC + 2));
        pp[tid] = m;
        pp[kHg + tid] = l;
      }
    }
    bar_softmax();
    tc_fence_after();
    const bool have = ok && c1 > c0;
    float* po = single ? nullptr
                       : P.part + ((size_t)stream * P.nsplit + split) * (kHg * (kC + 2)) + 2 * kHg;
    __nv_bfloat16* out =
        single ? static_cast<__nv_bfloat16*>(a.out) + ((size_t)bt * a.H + h0) * kC : nullptr;
    // O^T slice by slice (dims 128 sl + tid), G heads per TMEM load: all 64 with 64-row
    // chunks; 16 with 128-row chunks, where four smaller loads between the stores measured
    // faster (the one-chunk CTAs of the sparse decodes)
    constexpr int G = kRows == 64 ? 64 : 16;
#pragma unroll 1
    for (int cg = 0; cg < 4 * (64 / G); ++cg) {
      const int sl = cg / (64 / G), hb = G * (cg % (64 / G));
      uint32_t o[G];
      if (have) {
        if constexpr (G == 64) tmem_ld_32x32b_x64(lane_base + kColO + 64 * sl, o);
        else tmem_ld_x16(lane_base + kColO + 64 * sl + hb, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = 0u;
      }
      const int d = 128 * sl + tid;
      if (single) {
        float cs = 1.f, sn = 0.f;
        const bool rot = d >= r0;
        if (rot) {
          cs = S.cs[(d - r0) >> 1];
          sn = -S.sn[(d - r0) >> 1];  // rotation by -t
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float y = __uint_as_float(o[h]) * S.fin[hb + h];
          const float yp = __shfl_xor_sync(0xffffffffu, y, 1);
          float z = y;
          if (rot) z = (d & 1) == 0 ? y * cs - yp * sn : yp * sn + y * cs;
          out[(size_t)(hb + h) * kC + d] = __float2bfloat16_rn(z);
        }
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) po[(size_t)(hb + h) * kC + d] = __uint_as_float(o[h]);
      }
    }
  } else {
    // ------------------------------ MMA issuer (warp 4) ------------------------------
    const uint32_t idS = idesc_f16(1, kHg, kRows);              // M = 64, N = kRows, K-major
    const uint32_t idO = idesc_f16(1, 128, kHg) | (1u << 15);   // M = 128 dims; A MN-major
    // Descriptors are formed once; a step adds its operand's byte offset / 16 to the start
    // address field (every operand lies below 256 KB, so the 14-bit field never carries), and
    // the loops are unrolled, so issuing an MMA costs a few instructions.
    const uint64_t dq = smem_desc(smem_u32(base + kOffQ), 16, 1024, kLayoutSw128);
    bool ok = true;
    for (int j = c0; j < c1 && ok; ++j) {
      const uint32_t it = (uint32_t)(j - c0);
      const int slot = (int)(it % kBuf);
      const uint32_t ph = (it / kBuf) & 1;
      const uint32_t kv = smem_u32(base + kOffKV + slot * L::kSlotKV);
      const uint64_t dk = smem_desc(kv, 16, 1024, kLayoutSw128);           // K-major rows
      const uint64_t dv = smem_desc(kv, kRows * 128, 1024, kLayoutSw128);  // the same, MN-major
      const uint64_t dp = smem_desc(smem_u32(base + kOffP + slot * L::kSlotP), 16, 1024,
                                    kLayoutSw128);
      const uint32_t scol = tmem + kColS + (kBuf == 2 ? 64u * slot : 0u);
      ok = __all_sync(0xffffffffu, mbar_wait(&S.kv_full[slot], ph, kErrKvFull));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        // K = 512 in steps of 16: four steps per 64-dim atom. The atom loop is unrolled
        // for 64-row chunks (a CTA walks many, so the code is warm) and kept rolled for
        // 128-row chunks (typically one per CTA, where fetching a longer body costs more).
#pragma unroll(kRows == 64 ? 8 : 1)
        for (int atom = 0; atom < 8; ++atom) {
#pragma unroll
          for (int kq = 0; kq < 4; ++kq)
            mma_f16(scol, dq + ((atom * (kHg * 128) + kq * 32) >> 4),
                    dk + ((atom * (kRows * 128) + kq * 32) >> 4), idS,
                    (atom | kq) != 0 ? 1u : 0u);
        }
        mma_commit(&S.s_full[slot]);
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, mbar_wait(&S.p_full[slot], ph, kErrPFull));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        // K = kRows rows in steps of 16; the four O^T slices are independent accumulators,
        // issued in turn
#pragma unroll(kRows == 64 ? 4 : 1)
        for (int kk = 0; kk < kRows / 16; ++kk) {
#pragma unroll
          for (int sl = 0; sl < 4; ++sl)
            mma_f16(tmem + kColO + 64 * sl, dv + ((sl * 2 * (kRows * 128) + kk * 2048) >> 4),
                    dp + (((kk >> 2) * (kHg * 128) + (kk & 3) * 32) >> 4), idO,
                    (j > c0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&S.kv_free[slot]);
      }
      __syncwarp();
    }
    if (lane == 0) {  // nothing this thread issued is in flight once `done` fires
      mma_commit(&S.done);
      mbar_wait(&S.done, 0, kErrKvFree);
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the partials of each stream (fixed split order), add the sink, rotate by -t.
__global__ void __launch_bounds__(256) k_mqa_combine(MqaTcParams P) {
  pdl_wait();
  pdl_trigger();
  const MqaArgs& a = P.a;
  const int stream = blockIdx.x, h = blockIdx.y;
  const int bt = stream / P.G, g = stream % P.G;
  const int64_t t = a.q_pos[bt];
  const int tid = threadIdx.x;
  const size_t stride = kHg * (kC + 2);
  const float* base = P.part + (size_t)stream * P.nsplit * stride;
  constexpr int kMaxSplit = 32;  // choose_nsplit never exceeds this
  constexpr int kFirst = 16;     // splits whose (m, l, O) loads go out in the first round
  const int ns = P.nsplit;
  const int d = 2 * tid;
  float ms[kMaxSplit], lv[kFirst];
  float2 ov[kFirst];
#pragma unroll
  for (int sp = 0; sp < kMaxSplit; ++sp) ms[sp] = sp < ns ? base[sp * stride + h] : -INFINITY;
#pragma unroll
  for (int sp = 0; sp < kFirst; ++sp) {  // issued before the max is known: one round trip
    const float* pp = base + sp * stride;
    lv[sp] = sp < ns ? pp[kHg + h] : 0.f;
    ov[sp] = sp < ns ? *reinterpret_cast<const float2*>(pp + 2 * kHg + (size_t)h * kC + d)
                     : make_float2(0.f, 0.f);
  }
  float M = -INFINITY;
#pragma unroll
  for (int sp = 0; sp < kMaxSplit; ++sp) M = fmaxf(M, ms[sp]);
  const float zs = a.sink ? a.sink[g * kHg + h] : -INFINITY;
  const float Mt = fmaxf(M, zs);
  float l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
  for (int sp = 0; sp < kFirst; ++sp) {  // fixed split order: deterministic
    if (sp < ns && ms[sp] != -INFINITY) {
      const float f = expf(ms[sp] - Mt);
      l = fmaf(lv[sp], f, l);
      o0 = fmaf(ov[sp].x, f, o0);
      o1 = fmaf(ov[sp].y, f, o1);
    }
  }
  for (int sp = kFirst; sp < ns; ++sp) {  // more splits than the first round covers
    const float* pp = base + sp * stride;
    const float m = pp[h];  // reloaded: indexing ms here would put it in local memory
    if (m != -INFINITY) {
      const float f = expf(m - Mt);
      l = fmaf(pp[kHg + h], f, l);
      const float2 o = *reinterpret_cast<const float2*>(pp + 2 * kHg + (size_t)h * kC + d);
      o0 = fmaf(o.x, f, o0);
      o1 = fmaf(o.y, f, o1);
    }
  }
  float y0 = 0.f, y1 = 0.f;
  const float den = l + (zs == -INFINITY ? 0.f : expf(zs - Mt));
  if (l > 0.f) {
    y0 = o0 / den;
    y1 = o1 / den;
  }
  const int r = a.rope_dims, r0 = kC - r;
  if (d >= r0) {
    float cs, sn;
    rope_angle_cs(-(double)t, P.inv_freq[(d - r0) >> 1], &cs, &sn);
    const float u0 = y0 * cs - y1 * sn, u1 = y0 * sn + y1 * cs;
    y0 = u0;
    y1 = u1;
  }
  __nv_bfloat16* out =
      static_cast<__nv_bfloat16*>(a.out) + ((size_t)bt * a.H + g * kHg + h) * kC + d;
  *reinterpret_cast<__nv_bfloat162*>(out) = __floats2bfloat162_rn(y0, y1);
}

// bf16 rows of c = 512 values; box = one 128B swizzle atom (64 values) x box_rows rows
bool make_map_rows(CUtensorMap* m, const void* ptr, int64_t rows, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn || ptr == nullptr || rows < box_rows || rows >= (1ll << 31)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kC, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kC * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// CTAs per stream for chunks of R rows: as many as fill the SMs, at most one per chunk of
// the longest list, at most 32.
int splits_for(const MqaArgs& a, int R) {
  const int64_t streams = (int64_t)a.B * a.T * (a.H / kHg);
  const int64_t rows_max = (a.k > 0 ? a.k : a.n_cap) + a.n_win;
  const int64_t chunks_max = (rows_max + R - 1) / R;
  int64_t ns = device_sm_count() / (streams > 0 ? streams : 1);
  if (ns < 1) ns = 1;
  if (ns > chunks_max) ns = chunks_max > 0 ? chunks_max : 1;
  if (ns > 32) ns = 32;
  return (int)ns;
}

// Rows per chunk: 64, with two buffers, when a CTA walks two or more chunks of 128 (dense
// HCA lists, prefill: the next chunk's rows land during this one's softmax), or when
// 64-row chunks spread a short list over more CTAs and at most 12 partial states per
// stream (Flash decode: 10 CTAs of one chunk each instead of 5); otherwise 128 with one
// buffer (Pro decode, where 64-row chunks would make 18 partials per stream and the merge
// measured slower than the shorter chain saves).
int choose_rows(const MqaArgs& a) {
  const int64_t rows_max = (a.k > 0 ? a.k : a.n_cap) + a.n_win;
  const int64_t chunks = (rows_max + 127) / 128;
  const int ns = splits_for(a, 128);
  if ((chunks + ns - 1) / ns >= 2) return 64;
  const int ns64 = splits_for(a, 64);
  return ns64 > ns && ns64 <= 12 ? 64 : 128;
}

int choose_nsplit(const MqaArgs& a) { return splits_for(a, choose_rows(a)); }

}  // namespace

bool mqa_tc_supported(const MqaArgs& a, bool bf16) {
  const bool kv_ok = a.kv_scale == nullptr ||
                     (a.rope_dims > 0 && a.rope_dims < kC && a.rope_dims % 16 == 0);
  return bf16 && a.c == kC && a.H % kHg == 0 && a.rope_dims <= kC && a.rope_dims % 2 == 0 &&
         a.rope_dims / 2 <= 256 && kv_ok;
}

size_t mqa_tc_workspace_bytes(const MqaArgs& a) {
  const int ns = choose_nsplit(a);
  if (ns <= 1) return 0;
  const size_t streams = (size_t)a.B * a.T * (a.H / kHg);
  return streams * ns * kHg * (kC + 2) * sizeof(float);
}

cudaError_t launch_mqa_tc(const MqaArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
  MqaTcParams P;
  P.a = a;
  P.G = a.H / kHg;
  P.nsplit = choose_nsplit(a);
  P.part = P.nsplit > 1 ? static_cast<float*>(ws) : nullptr;
  for (int p = 0; p < kMaxPairs; ++p)
    P.inv_freq[p] = p < a.rope_dims / 2 ? rope_inv_freq(p, a.rope_dims, (double)a.rope_base) : 0.0;
  CUtensorMap tm_kv, tm_win;
  memset(&tm_kv, 0, sizeof(tm_kv));
  memset(&tm_win, 0, sizeof(tm_win));
  const bool mixed = a.kv_scale != nullptr;    // mixed-precision cache rows
  const bool paged = a.page_table != nullptr;  // cache rows through the page table
  const int rows = choose_rows(a);
  // cache rows come by TMA only when they are contiguous bf16 rows
  P.tma_kv =
      !mixed && !paged && make_map_rows(&tm_kv, a.kv, (int64_t)a.B * a.n_cap, rows) ? 1 : 0;
  // window rows by TMA only from a linear window buffer (a ring wraps)
  P.tma_win =
      a.win_pos0 != nullptr && make_map_rows(&tm_win, a.win, (int64_t)a.B * a.l_raw, rows) ? 1 : 0;
  if (P.nsplit > 1 && ws_bytes < mqa_tc_workspace_bytes(a)) return cudaErrorInvalidValue;
  const int64_t streams = (int64_t)a.B * a.T * P.G;
  auto kern = rows == 64
                  ? (mixed ? (paged ? k_mqa_tc<true, true, 64> : k_mqa_tc<true, false, 64>)
                           : (paged ? k_mqa_tc<false, true, 64> : k_mqa_tc<false, false, 64>))
                  : (mixed ? (paged ? k_mqa_tc<true, true, 128> : k_mqa_tc<true, false, 128>)
                           : (paged ? k_mqa_tc<false, true, 128> : k_mqa_tc<false, false, 128>));
  const size_t smem =
      1024 + (rows == 64 ? Lay<64>::kOffEnd +
                               (mixed ? sizeof(SmemT<true, 64>) : sizeof(SmemT<false, 64>))
                         : Lay<128>::kOffEnd +
                               (mixed ? sizeof(SmemT<true, 128>) : sizeof(SmemT<false, 128>)));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  e = launch(a.chained, kern, dim3((unsigned)(streams * P.nsplit)), dim3(kThreads), smem, st,
             tm_kv, tm_win, P);
  if (e != cudaSuccess || P.nsplit == 1) return e;
  return launch(true, k_mqa_combine, dim3((unsigned)streams, kHg), dim3(256), 0, st, P);
}

cudaError_t mqa_tc_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, tc::g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));
}

}  // namespace csa
