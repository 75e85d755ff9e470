// Stage 3 for few long rows (decode): top-k of each query's scores over up to ~10^6
// entries, spread over many CTAs.
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): the top-k selector keeps the k entries with the
// largest index scores. Result order: (score desc, index asc); -1 past the visible count.
//
// 1. A 4096-bin histogram of the top 12 bits of every score's order-preserving key (fused
//    into the tensor-core indexer's epilogue, or k_topk_hist here).
// 2. k_topk_filter: every CTA loads its slice of the row, finds the bin T holding the k-th
//    largest key, and appends the entries of bins > T to the "sure" list (fewer than k in
//    all) and those of bin T to the "boundary" list, with one atomic per list per CTA.
// 3. k_topk_rank: every candidate (sure or boundary) is identified by the 64-bit value
//    (key << 32 | ~index), unique per entry, larger = better (score desc, index asc). Its
//    place in the result is the number of candidates with a larger value (for a boundary
//    entry: ns + those in the boundary list), counted by many CTAs per query, so no select
//    or sort runs in one CTA; a candidate whose place is below min(k, n_vis) is written
//    there. With more than 2048 boundary entries (heavy
//    ties) one CTA per query instead radix-selects the boundary entries it needs and merge
//    sorts the winners. Either way the result depends on the scores only.
#include "common.cuh"
#include "internal.h"
#include "qhat.cuh"

namespace csa {

namespace {

constexpr int kBins = 4096;
constexpr int kFThreads = 256;
constexpr int kWarps = kFThreads / 32;
constexpr int kDigitBits = 11;   // radix-select digit width
constexpr int kDigits = 1 << kDigitBits;
constexpr int kRankBnd = 2048;                 // boundary entries the rank path takes
constexpr int kRankPerCta = 32;                // candidates ranked by one CTA

__device__ __forceinline__ int64_t visible(const int64_t* q_pos, int q, int m, int64_t n_cap) {
  const int64_t t = q_pos[q];
  return t < 0 ? 0 : (t / m < n_cap ? t / m : n_cap);
}

// value ordering "better first" = larger v; the sort key (ascending) is ~v
__device__ __forceinline__ uint64_t sel_value(uint32_t key, uint32_t idx) {
  return ((uint64_t)key << 32) | (uint64_t)(0xffffffffu - idx);
}

// Ascending merge sort of arr[0..P), P = E * kFThreads, with `tmp` (P entries) as the
// second buffer; returns the buffer holding the result. Each thread first sorts E elements
// in registers (odd-even transposition), then every level merges pairs of sorted runs:
// thread t writes outputs E*t .. E*t+E-1 of its pair, locating its start by a binary
// search along the merge path (ties go to the left run, so equal values are handled).
// About log2(P/E) barriers in all: the latency of a long network of dependent
// compare-exchange stages is what this replaces.
template <int E>
__device__ uint64_t* merge_sort(uint64_t* arr, uint64_t* tmp) {
  constexpr int P = E * kFThreads;
  const int tid = threadIdx.x;
  {
    uint64_t x[E];
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = arr[E * tid + e];
#pragma unroll
    for (int round = 0; round < E; ++round) {
#pragma unroll
      for (int e = round & 1; e + 1 < E; e += 2) {
        const uint64_t u = x[e], v = x[e + 1];
        x[e] = u < v ? u : v;
        x[e + 1] = u < v ? v : u;
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) arr[E * tid + e] = x[e];
  }
  __syncthreads();
  uint64_t* src = arr;
  uint64_t* dst = tmp;
#pragma unroll 1
  for (int L = E; L < P; L <<= 1) {
    const int out0 = E * tid;
    const int base = out0 & ~(2 * L - 1);
    const int d = out0 - base;  // outputs of the merged pair before this thread's first
    const uint64_t* A = src + base;
    const uint64_t* B = A + L;
    int lo = d > L ? d - L : 0, hi = d < L ? d : L;
    while (lo < hi) {  // i = how many of the first d outputs come from A
      const int mid = (lo + hi) >> 1;
      if (A[mid] <= B[d - mid - 1]) lo = mid + 1; else hi = mid;
    }
    int i = lo, j = d - lo;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const uint64_t av = i < L ? A[i] : ~0ull, bv = j < L ? B[j] : ~0ull;
      const bool take_a = j >= L || (i < L && av <= bv);
      dst[out0 + e] = take_a ? av : bv;
      i += take_a;
      j += !take_a;
    }
    __syncthreads();
    uint64_t* t = src;
    src = dst;
    dst = t;
  }
  return src;
}

// Row q of the scores, in their storage type (fp32, or bf16 for the selector on BF16 index
// scores).
template <typename TS>
__device__ __forceinline__ const TS* score_row(const TopkDecodeArgs& a, int q) {
  if constexpr (sizeof(TS) == 4) return a.scores + (size_t)q * a.n_cap;
  else return static_cast<const TS*>(a.scores16) + (size_t)q * a.n_cap;
}

template <typename TS>
__global__ void __launch_bounds__(kFThreads) k_topk_hist(TopkDecodeArgs a) {
  __shared__ int h[kBins];
  const int q = blockIdx.y;
  const int64_t n = visible(a.q_pos, q, a.m, a.n_cap);
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t lo = n * blockIdx.x / gridDim.x, hi = n * (blockIdx.x + 1) / gridDim.x;
  const TS* sc = score_row<TS>(a, q);
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x)
    atomicAdd(&h[float_key(ld_score(sc, i)) >> 20], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += blockDim.x)
    if (h[i]) atomicAdd(&a.hist[(size_t)q * kBins + i], h[i]);
}

// Exclusive block scan of two counts per thread; returns the offsets and the block
// totals. `ws` is shared scratch of 2 * kWarps ints. Ends with a barrier.
__device__ __forceinline__ void block_scan2(int c0, int c1, int* ws, int* o0, int* o1, int* t0,
                                            int* t1) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int i0 = c0, i1 = c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x0 = __shfl_up_sync(0xffffffffu, i0, o), x1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += x0;
      i1 += x1;
    }
  }
  if (lane == 31) {
    ws[wid] = i0;
    ws[kWarps + wid] = i1;
  }
  __syncthreads();
  int p0 = 0, p1 = 0, s0 = 0, s1 = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int v0 = ws[w], v1 = ws[kWarps + w];
    if (w < wid) {
      p0 += v0;
      p1 += v1;
    }
    s0 += v0;
    s1 += v1;
  }
  *o0 = p0 + i0 - c0;
  *o1 = p1 + i1 - c1;
  *t0 = s0;
  *t1 = s1;
  __syncthreads();
}

// zero n0 + n1 int4 words of two ranges (histograms and counters of a call), in stream order
// Triggers before it waits: the next kernel (the indexer) may then start its set-up while
// this one waits, which is safe because that set-up reads nothing a predecessor writes.
__global__ void __launch_bounds__(256) k_zero(int4* p0, int n0, int4* p1, int n1) {
  pdl_trigger();
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n0 + n1; i += gridDim.x * blockDim.x) {
    if (i < n0) p0[i] = make_int4(0, 0, 0, 0);
    else p1[i - n0] = make_int4(0, 0, 0, 0);
  }
}

template <typename TS>
__global__ void __launch_bounds__(kFThreads, 2) k_topk_filter(TopkDecodeArgs a) {
  __shared__ int wsum[2 * kWarps];
  __shared__ int s_bin, s_base_s, s_base_b;
  __shared__ float s_cs[256], s_sn[256];
  if (a.qj.qhat != nullptr) {  // this CTA's share of the query's heads
    const int hq = blockIdx.y;
    qhat_rows(a.qj, hq, (double)a.q_pos[hq], a.qj.H * blockIdx.x / gridDim.x,
              a.qj.H * (blockIdx.x + 1) / gridDim.x, s_cs, s_sn);
  }
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.y, tid = threadIdx.x;
  const int nslice = gridDim.x;
  const int64_t n = visible(a.q_pos, q, a.m, a.n_cap);
  const int k = a.k;
  int* cnt = a.cnt + 4 * q;  // sure count, boundary count
  uint64_t* sure = a.list + (size_t)q * (a.n_cap + k);
  uint64_t* bnd = sure + k;

  // ---- this CTA's slice: first batch of loads in flight before the threshold is known ----
  const int64_t lo = n * blockIdx.x / nslice, hi = n * (blockIdx.x + 1) / nslice;
  const TS* sc = score_row<TS>(a, q);
  constexpr int kBatch = 16;  // loads in flight per thread
  float f[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const int64_t i = lo + j * kFThreads + tid;
    f[j] = i < hi ? ld_score(sc, i) : 0.f;
  }

  // ---- threshold bin: the bin holding the k-th largest key ----
  if (tid == 0) s_bin = -1;
  if (n > k) {
    // thread t owns bins 4095-16t .. 4080-16t (descending), read as four int4
    const int4* hp =
        reinterpret_cast<const int4*>(a.hist + (size_t)q * kBins + kBins - 16 - 16 * tid);
    int v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int4 x = hp[3 - j];
      v[4 * j] = x.w;
      v[4 * j + 1] = x.z;
      v[4 * j + 2] = x.y;
      v[4 * j + 3] = x.x;
    }
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) sum += v[j];
    int off, dummy, tot, tot2;
    block_scan2(sum, 0, wsum, &off, &dummy, &tot, &tot2);
    int above = off;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (above < k && above + v[j] >= k) s_bin = kBins - 1 - 16 * tid - j;
      above += v[j];
    }
  }
  __syncthreads();
  const int T = s_bin;  // -1: every visible entry is selected

  // ---- append: sure entries (bin > T) and boundary entries (bin == T), one atomic each ----
  for (int64_t base = lo; base < hi; base += kBatch * kFThreads) {
    if (base != lo) {
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int64_t i = base + j * kFThreads + tid;
        f[j] = i < hi ? ld_score(sc, i) : 0.f;
      }
    }
    uint32_t fs = 0, fb = 0;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t i = base + j * kFThreads + tid;
      const int bin = (int)(float_key(f[j]) >> 20);
      fs |= (uint32_t)(i < hi && bin > T) << j;
      fb |= (uint32_t)(i < hi && bin == T) << j;
    }
    int os, ob, ts, tb;
    block_scan2(__popc(fs), __popc(fb), wsum, &os, &ob, &ts, &tb);
    if (ts + tb == 0) continue;  // uniform
    if (tid == 0) {
      s_base_s = ts ? atomicAdd(&cnt[0], ts) : 0;
      s_base_b = tb ? atomicAdd(&cnt[1], tb) : 0;
    }
    __syncthreads();
    os += s_base_s;
    ob += s_base_b;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const uint64_t v = sel_value(float_key(f[j]), (uint32_t)(base + j * kFThreads + tid));
      if (fs >> j & 1) {
        if (os < k) sure[os] = v;
        ++os;
      }
      if (fb >> j & 1) {
        if (ob < a.n_cap) bnd[ob] = v;
        ++ob;
      }
    }
    __syncthreads();  // s_base_* are reused by the next batch
  }

}

__global__ void __launch_bounds__(kFThreads) k_topk_rank(TopkDecodeArgs a) {
  __shared__ __align__(16) uint64_t cand[kMaxTopk + kRankBnd];  // fallback: pairs + bcache
  __shared__ int dh[kDigits];
  __shared__ int wsum[2 * kWarps];
  __shared__ int part[kWarps][kRankPerCta];
  __shared__ uint32_t s_digit;
  __shared__ int s_dabove, s_fill, s_fill_exact;
  pdl_wait();
  pdl_trigger();
  uint64_t* pairs = cand;
  uint64_t* bcache = cand + kMaxTopk;
  const int q = blockIdx.y, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t n = visible(a.q_pos, q, a.m, a.n_cap);
  const int k = a.k;
  const int nsel = (int)(n < k ? n : k);
  const int* cnt = a.cnt + 4 * q;
  const uint64_t* sure = a.list + (size_t)q * (a.n_cap + k);
  const uint64_t* bnd = sure + k;
  int32_t* out = a.out_idx + (size_t)q * k;
  const int ns = min(__ldcg(&cnt[0]), k);
  const int nb = (int)min((int64_t)__ldcg(&cnt[1]), a.n_cap);

  if (nb <= kRankBnd) {
    // ---- rank path: every sure value is above every boundary value, so a sure entry's
    //      place is its rank among the sure entries and a boundary entry's is ns + its
    //      rank among the boundary entries; CTAs take 32 entries of one list each ----
    const int cs = (ns + kRankPerCta - 1) / kRankPerCta;
    if (blockIdx.x == 0)
      for (int i = nsel + tid; i < k; i += kFThreads) out[i] = -1;
    const bool in_sure = (int)blockIdx.x < cs;
    const int C = in_sure ? ns : nb;
    const int c0 = (in_sure ? blockIdx.x : blockIdx.x - cs) * kRankPerCta;
    if (c0 >= C) return;
    const uint64_t* list = in_sure ? sure : bnd;
    const int place0 = in_sure ? 0 : ns;
    constexpr int kLoads = kRankBnd / kFThreads;
    uint64_t v[kLoads];
#pragma unroll
    for (int j = 0; j < kLoads; ++j) {
      const int c = tid + j * kFThreads;
      v[j] = c < C ? __ldcg(&list[c]) : 0ull;
    }
#pragma unroll
    for (int j = 0; j < kLoads; ++j) {
      const int c = tid + j * kFThreads;
      if (c < C) cand[c] = v[j];
    }
    __syncthreads();
    // lane = entry of this CTA, warp = a range of the list (broadcast reads)
    const int ci = c0 + lane;
    const uint64_t x = ci < C ? cand[ci] : ~0ull;
    const int j0 = (int)((int64_t)C * wid / kWarps), j1 = (int)((int64_t)C * (wid + 1) / kWarps);
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    int j = j0;
    for (; j + 4 <= j1; j += 4) {
      r0 += cand[j] > x;
      r1 += cand[j + 1] > x;
      r2 += cand[j + 2] > x;
      r3 += cand[j + 3] > x;
    }
    for (; j < j1; ++j) r0 += cand[j] > x;
    part[wid][lane] = (r0 + r1) + (r2 + r3);
    __syncthreads();
    if (wid == 0 && ci < C) {
      int rank = place0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) rank += part[w][lane];
      if (rank < nsel) out[rank] = (int32_t)(0xffffffffu - (uint32_t)(x & 0xffffffffu));
    }
    return;
  }

  // ---- heavy ties (many boundary entries): one CTA selects and sorts ----
  if (blockIdx.x != 0) return;
  const int T = (int)(__ldcg(&bnd[0]) >> 52);  // every boundary value shares bin T
  int kk = nsel - ns;  // still to take from the boundary list
  if (kk < 0) kk = 0;
  if (kk > nb) kk = nb;
  for (int i = tid; i < ns; i += kFThreads) pairs[i] = ~__ldcg(&sure[i]);
  if (tid == 0) s_fill = ns;
  __syncthreads();
  if (kk > 0) {
    uint64_t thr = 0;  // take every boundary value >= thr
    if (kk < nb) {
      // every boundary value shares the top 12 key bits (bin T): radix-select below them
      uint64_t prefix = (uint64_t)T << 52, mask = (uint64_t)0xfff << 52;
      int need = kk;
      for (int hi_bit = 52; hi_bit > 0;) {
        const int width = hi_bit >= kDigitBits ? kDigitBits : hi_bit;
        const int shift = hi_bit - width;
        const uint64_t dmask = ((uint64_t)1 << width) - 1;
        for (int i = tid; i < kDigits; i += kFThreads) dh[i] = 0;
        if (tid == 0) s_fill_exact = 0;
        __syncthreads();
        for (int i = tid; i < nb; i += kFThreads) {
          const uint64_t v = __ldcg(&bnd[i]);
          if ((v & mask) == prefix) atomicAdd(&dh[(v >> shift) & dmask], 1);
        }
        __syncthreads();
        // thread t owns digits 2047-8t .. 2040-8t (descending)
        constexpr int kPer = kDigits / kFThreads;
        int c[kPer], sum = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          c[j] = dh[kDigits - 1 - kPer * tid - j];
          sum += c[j];
        }
        int off, dummy, tot, tot2;
        block_scan2(sum, 0, wsum, &off, &dummy, &tot, &tot2);
        int above = off;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          if (above < need && above + c[j] >= need) {
            s_digit = kDigits - 1 - kPer * tid - j;
            s_dabove = above;
            s_fill_exact = (above + c[j] == need);  // the digit's bucket is taken whole
          }
          above += c[j];
        }
        __syncthreads();
        prefix |= (uint64_t)s_digit << shift;
        mask |= dmask << shift;
        need -= s_dabove;
        const bool whole = s_fill_exact;
        __syncthreads();
        hi_bit = shift;
        if (whole) break;  // lower bits of prefix are zero: values >= prefix are exactly kk
      }
      thr = prefix;
    }
    for (int i = tid; i < nb; i += kFThreads) {
      const uint64_t v = __ldcg(&bnd[i]);
      if (v >= thr) {
        const int pos = atomicAdd(&s_fill, 1);
        if (pos < kMaxTopk) pairs[pos] = ~v;
      }
    }
  }
  __syncthreads();
  const int filled = min(s_fill, nsel);
  const int P = k <= kMaxTopk / 4 ? kMaxTopk / 4 : (k <= kMaxTopk / 2 ? kMaxTopk / 2 : kMaxTopk);
  for (int i = filled + tid; i < P; i += kFThreads) pairs[i] = ~0ull;
  __syncthreads();
  // bcache is free now: it is the merge sort's second buffer
  const uint64_t* sorted = P == kMaxTopk       ? merge_sort<kMaxTopk / kFThreads>(pairs, bcache)
                           : P == kMaxTopk / 2 ? merge_sort<kMaxTopk / 2 / kFThreads>(pairs, bcache)
                                               : merge_sort<kMaxTopk / 4 / kFThreads>(pairs, bcache);
  for (int i = tid; i < k; i += kFThreads)
    out[i] = i < filled ? (int32_t)(sorted[i] & 0xffffffffu) : -1;
}

}  // namespace

bool topk_decode_path(int B, int T, int64_t n_cap, int k) {
  return (int64_t)B * T <= 64 && n_cap >= 8192 && k <= kMaxTopk;
}

static size_t rup(size_t x) { return (x + 255) / 256 * 256; }

size_t topk_decode_ws_bytes(int B, int T, int64_t n_cap, int k) {
  const size_t Q = (size_t)B * T;
  return rup(Q * kBins * 4) + rup(Q * 16) + rup(Q * ((size_t)n_cap + k) * 8);
}

TopkDecodeArgs topk_decode_args(const TopkArgs& t, void* ws) {
  TopkDecodeArgs a{};
  const size_t Q = (size_t)t.B * t.T;
  char* p = static_cast<char*>(ws);
  a.Q = (int)Q; a.m = t.m; a.k = t.k; a.n_cap = t.n_cap; a.scores = t.scores;
  a.scores16 = t.scores16;
  a.q_pos = t.q_pos; a.out_idx = t.out_idx; a.qj = t.qj;
  a.hist = reinterpret_cast<int*>(p);
  p += rup(Q * kBins * 4);
  a.cnt = reinterpret_cast<int*>(p);
  p += rup(Q * 16);
  a.list = reinterpret_cast<uint64_t*>(p);
  return a;
}

cudaError_t topk_decode_clear(const TopkDecodeArgs& a, cudaStream_t st) {
  // hist and the counters are adjacent at the start of the workspace
  const size_t bytes = rup((size_t)a.Q * kBins * 4) + rup((size_t)a.Q * 16);
  return launch_zero(a.hist, bytes, nullptr, 0, st);
}

cudaError_t launch_zero(void* p0, size_t b0, void* p1, size_t b1, cudaStream_t st) {
  const int n0 = (int)(b0 / 16), n1 = p1 ? (int)(b1 / 16) : 0;
  const int blocks = (n0 + n1 + 255) / 256;
  return launch(true, k_zero, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st,
                reinterpret_cast<int4*>(p0), n0, reinterpret_cast<int4*>(p1), n1);
}

cudaError_t launch_topk_decode(TopkDecodeArgs a, bool hist_ready, cudaStream_t st) {
  if (a.Q == 0) return cudaSuccess;
  int slices = (2 * 148) / a.Q;
  const int64_t max_slices = (a.n_cap + 2047) / 2048;
  if (slices > max_slices) slices = (int)max_slices;
  if (slices < 1) slices = 1;
  a.nslice = slices;
  if (!hist_ready) {
    const cudaError_t e = topk_decode_clear(a, st);
    if (e != cudaSuccess) return e;
    const cudaError_t eh =
        a.scores16 ? launch(false, k_topk_hist<__nv_bfloat16>, dim3(slices, a.Q), dim3(kFThreads),
                            0, st, a)
                   : launch(false, k_topk_hist<float>, dim3(slices, a.Q), dim3(kFThreads), 0, st, a);
    if (eh != cudaSuccess) return eh;
  }
  cudaError_t e =
      a.scores16
          ? launch(true, k_topk_filter<__nv_bfloat16>, dim3(slices, a.Q), dim3(kFThreads), 0, st, a)
          : launch(true, k_topk_filter<float>, dim3(slices, a.Q), dim3(kFThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  // enough CTAs for the sure list (< k) and the boundary list (<= kRankBnd) apart
  const int rank_ctas = (a.k + kRankPerCta - 1) / kRankPerCta + kRankBnd / kRankPerCta;
  return launch(true, k_topk_rank, dim3(rank_ctas, a.Q), dim3(kFThreads), 0, st, a);
}

}  // namespace csa
