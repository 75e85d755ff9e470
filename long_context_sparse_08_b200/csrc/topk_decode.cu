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
//    all) and those of bin T to the "boundary" list, with one atomic per list per CTA. The
//    last CTA of a query (atomic ticket) selects the remaining entries from the boundary
//    list by an exact radix select on the 64-bit value (key << 32 | ~index), which is
//    unique per entry, so ties resolve to the lower index, and sorts the winners. The
//    result depends on the scores only.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kBins = 4096;
constexpr int kFThreads = 256;
constexpr int kWarps = kFThreads / 32;
constexpr int kBndCache = 2048;  // boundary entries kept in shared memory for the final pass
constexpr int kDigitBits = 11;   // radix-select digit width
constexpr int kDigits = 1 << kDigitBits;

__device__ __forceinline__ int64_t visible(const int64_t* q_pos, int q, int m, int64_t n_cap) {
  const int64_t t = q_pos[q];
  return t < 0 ? 0 : (t / m < n_cap ? t / m : n_cap);
}

// value ordering "better first" = larger v; the sort key (ascending) is ~v
__device__ __forceinline__ uint64_t sel_value(uint32_t key, uint32_t idx) {
  return ((uint64_t)key << 32) | (uint64_t)(0xffffffffu - idx);
}

// Ascending bitonic sort of arr[0..P) (P a power of two, 1024 or 2048), with kFThreads
// threads. Thread t keeps elements E*t .. E*t+E-1 in registers; exchanges at distance < E
// stay inside a thread, those below 32*E go through warp shuffles, and only the wider ones
// through shared memory (one barrier each). Leaves the sorted values in arr.
template <int E>
__device__ void bitonic_sort_regs(uint64_t* arr) {
  constexpr int P = E * kFThreads;
  const int tid = threadIdx.x;
  uint64_t x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = arr[E * tid + e];
  bool in_regs = true;
#pragma unroll 1
  for (int size = 2; size <= P; size <<= 1) {
#pragma unroll 1
    for (int s = size >> 1; s > 0; s >>= 1) {
      if (s >= 32 * E) {  // partner in another warp
        if (in_regs) {
#pragma unroll
          for (int e = 0; e < E; ++e) arr[E * tid + e] = x[e];
          __syncthreads();
          in_regs = false;
        }
        for (int i = tid; i < (P >> 1); i += kFThreads) {
          const int lo = 2 * i - (i & (s - 1)), hi = lo + s;
          const bool asc = (lo & size) == 0;
          const uint64_t u = arr[lo], v = arr[hi];
          if ((u > v) == asc) {
            arr[lo] = v;
            arr[hi] = u;
          }
        }
        __syncthreads();
        continue;
      }
      if (!in_regs) {
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = arr[E * tid + e];
        in_regs = true;
      }
      if (s >= E) {  // partner element i ^ s sits in lane ^ (s / E), same slot
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = E * tid + e;
          const uint64_t y = __shfl_xor_sync(0xffffffffu, x[e], s / E);
          const bool asc = (i & size) == 0, lo = (i & s) == 0;
          const bool take_min = asc == lo;
          x[e] = take_min ? (x[e] < y ? x[e] : y) : (x[e] < y ? y : x[e]);
        }
      } else {  // partner inside this thread (s = E/2 .. 1; indices stay compile-time)
#pragma unroll
        for (int sc = E / 2; sc > 0; sc >>= 1) {
          if (sc != s) continue;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            if ((e & sc) == 0) {
              const bool asc = ((E * tid + e) & size) == 0;
              const uint64_t u = x[e], v = x[e + sc];
              if ((u > v) == asc) {
                x[e] = v;
                x[e + sc] = u;
              }
            }
          }
        }
      }
    }
  }
  if (in_regs) {  // each thread stores back the slots it loaded: no cross-thread hazard
#pragma unroll
    for (int e = 0; e < E; ++e) arr[E * tid + e] = x[e];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kFThreads) k_topk_hist(TopkDecodeArgs a) {
  __shared__ int h[kBins];
  const int q = blockIdx.y;
  const int64_t n = visible(a.q_pos, q, a.m, a.n_cap);
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t lo = n * blockIdx.x / gridDim.x, hi = n * (blockIdx.x + 1) / gridDim.x;
  const float* sc = a.scores + (size_t)q * a.n_cap;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x)
    atomicAdd(&h[float_key(sc[i]) >> 20], 1);
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

__global__ void __launch_bounds__(kFThreads, 2) k_topk_filter(TopkDecodeArgs a) {
  __shared__ __align__(16) uint64_t bcache[kBndCache];
  __shared__ uint64_t pairs[kMaxTopk];
  __shared__ int dh[kDigits];
  __shared__ int wsum[2 * kWarps];
  __shared__ int s_bin, s_last, s_base_s, s_base_b;
  __shared__ uint32_t s_digit;
  __shared__ int s_dabove, s_fill, s_fill_exact;
  const int q = blockIdx.y, tid = threadIdx.x;
  const int nslice = gridDim.x;
  const int64_t n = visible(a.q_pos, q, a.m, a.n_cap);
  const int k = a.k;
  const int nsel = (int)(n < k ? n : k);
  int* cnt = a.cnt + 4 * q;  // sure count, boundary count, ticket
  uint64_t* sure = a.list + (size_t)q * (a.n_cap + k);
  uint64_t* bnd = sure + k;

  // ---- this CTA's slice: first batch of loads in flight before the threshold is known ----
  const int64_t lo = n * blockIdx.x / nslice, hi = n * (blockIdx.x + 1) / nslice;
  const float* sc = a.scores + (size_t)q * a.n_cap;
  constexpr int kBatch = 16;  // loads in flight per thread
  float f[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const int64_t i = lo + j * kFThreads + tid;
    f[j] = i < hi ? sc[i] : 0.f;
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
        f[j] = i < hi ? sc[i] : 0.f;
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

  // ---- the last CTA of this query finishes the selection ----
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(&cnt[2], 1) == nslice - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int ns = min(__ldcg(&cnt[0]), k);
  const int nb = (int)min((int64_t)__ldcg(&cnt[1]), a.n_cap);
  int kk = nsel - ns;  // still to take from the boundary list
  if (kk < 0) kk = 0;
  if (kk > nb) kk = nb;
  const bool cached = nb <= kBndCache;
  {  // both lists into shared memory, all loads issued before the stores
    constexpr int kS = kMaxTopk / kFThreads, kB = kBndCache / kFThreads;
    uint64_t sv[kS], bv[kB];
#pragma unroll
    for (int j = 0; j < kS; ++j) {
      const int e = tid + j * kFThreads;
      sv[j] = e < ns ? __ldcg(&sure[e]) : 0ull;
    }
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int e = tid + j * kFThreads;
      bv[j] = (kk > 0 && cached && e < nb) ? __ldcg(&bnd[e]) : 0ull;
    }
#pragma unroll
    for (int j = 0; j < kS; ++j) {
      const int e = tid + j * kFThreads;
      if (e < ns) pairs[e] = ~sv[j];
    }
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int e = tid + j * kFThreads;
      if (kk > 0 && cached && e < nb) bcache[e] = bv[j];
    }
  }
  if (tid == 0) s_fill = ns;
  __syncthreads();
  const uint64_t* L = cached ? bcache : bnd;
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
          const uint64_t v = cached ? L[i] : __ldcg(&L[i]);
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
      const uint64_t v = cached ? L[i] : __ldcg(&L[i]);
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
  if (P == kMaxTopk)
    bitonic_sort_regs<kMaxTopk / kFThreads>(pairs);
  else if (P == kMaxTopk / 2)
    bitonic_sort_regs<kMaxTopk / 2 / kFThreads>(pairs);
  else
    bitonic_sort_regs<kMaxTopk / 4 / kFThreads>(pairs);
  int32_t* out = a.out_idx + (size_t)q * k;
  for (int i = tid; i < k; i += kFThreads)
    out[i] = i < filled ? (int32_t)(pairs[i] & 0xffffffffu) : -1;
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
  a.q_pos = t.q_pos; a.out_idx = t.out_idx;
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
  return cudaMemsetAsync(a.hist, 0, bytes, st);
}

cudaError_t launch_topk_decode(TopkDecodeArgs a, bool hist_ready, cudaStream_t st) {
  if (a.Q == 0) return cudaSuccess;
  int slices = (2 * 148) / a.Q;
  const int64_t max_slices = (a.n_cap + 2047) / 2048;
  if (slices > max_slices) slices = (int)max_slices;
  if (slices < 1) slices = 1;
  a.nslice = slices;
  if (!hist_ready) {
    cudaError_t e = topk_decode_clear(a, st);
    if (e != cudaSuccess) return e;
    k_topk_hist<<<dim3(slices, a.Q), kFThreads, 0, st>>>(a);
  }
  k_topk_filter<<<dim3(slices, a.Q), kFThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
