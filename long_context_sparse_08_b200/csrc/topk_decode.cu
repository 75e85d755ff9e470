// Stage 3 for few long rows (decode): top-k of each query's scores over up to ~10^6
// entries, spread over many CTAs.
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): the top-k selector keeps the k entries with the
// largest index scores. Result order: (score desc, index asc); -1 past the visible count.
//
// 1. A 4096-bin histogram of the top 12 bits of every score's order-preserving key (fused
//    into the tensor-core indexer's epilogue, or k_topk_hist here).
// 2. k_topk_filter: every CTA finds the bin T holding the k-th largest key and appends, from
//    its slice of the row, the entries of bins > T to the "sure" list (fewer than k) and
//    those of bin T to the "boundary" list. The last CTA of a query (atomic ticket) selects
//    the remaining entries from the boundary list by an exact radix select on the 64-bit
//    value (key << 32 | ~index), which is unique per entry, so ties resolve to the lower
//    index; then it sorts the k winners. The result depends on the scores only.
#include "common.cuh"
#include "internal.h"

namespace csa {

namespace {

constexpr int kBins = 4096;
constexpr int kFThreads = 512;
constexpr int kBndCache = 2048;  // boundary entries kept in shared memory for the final pass

__device__ __forceinline__ int64_t visible(const int64_t* q_pos, int q, int m, int64_t n_cap) {
  const int64_t t = q_pos[q];
  return t < 0 ? 0 : (t / m < n_cap ? t / m : n_cap);
}

// value ordering "better first" = larger v; the sort key (ascending) is ~v
__device__ __forceinline__ uint64_t sel_value(uint32_t key, uint32_t idx) {
  return ((uint64_t)key << 32) | (uint64_t)(0xffffffffu - idx);
}

__device__ void bitonic_sort_u64(uint64_t* arr, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (P >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint64_t x = arr[lo], y = arr[hi];
        if ((x > y) == asc) {
          arr[lo] = y;
          arr[hi] = x;
        }
      }
      __syncthreads();
    }
  }
}

// warp-aggregated append of `v` to list[*counter] (capacity cap)
__device__ __forceinline__ void append(bool take, uint64_t v, int* counter, uint64_t* list,
                                       int cap) {
  const unsigned bal = __ballot_sync(0xffffffffu, take);
  if (bal == 0) return;
  const int lane = threadIdx.x & 31;
  int base = 0;
  if (lane == __ffs(bal) - 1) base = atomicAdd(counter, __popc(bal));
  base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
  if (take) {
    const int pos = base + __popc(bal & ((1u << lane) - 1u));
    if (pos < cap) list[pos] = v;
  }
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

__global__ void __launch_bounds__(kFThreads) k_topk_filter(TopkDecodeArgs a) {
  // the histogram is dead once the threshold bin is known; the final pass reuses it
  __shared__ __align__(16) uint64_t hbuf[kBndCache];
  static_assert(kBndCache * 8 == kBins * 4, "boundary cache aliases the histogram");
  int* h = reinterpret_cast<int*>(hbuf);
  uint64_t* bcache = hbuf;
  __shared__ int wsum[kFThreads / 32 + 1];
  __shared__ int s_bin, s_above, s_last;
  __shared__ uint64_t pairs[kMaxTopk];
  __shared__ int hist256[256];
  __shared__ uint32_t s_digit;
  __shared__ int s_dabove, s_fill, s_fill_exact;
  const int q = blockIdx.y, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t n = visible(a.q_pos, q, a.m, a.n_cap);
  const int k = a.k;
  const int nsel = (int)(n < k ? n : k);
  int* cnt = a.cnt + 4 * q;

  // ---- threshold bin: the bin holding the k-th largest key ----
  for (int i = tid; i < kBins; i += blockDim.x) h[i] = a.hist[(size_t)q * kBins + i];
  if (tid == 0) {
    s_bin = -1;
    s_above = 0;
  }
  __syncthreads();
  if (n > k) {
    int v[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // thread t owns bins 4095-8t .. 4088-8t (descending)
      v[j] = h[kBins - 1 - 8 * tid - j];
      sum += v[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    int wpre = 0;
    for (int w = 0; w < wid; ++w) wpre += wsum[w];
    int above = wpre + incl - sum;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (above < k && above + v[j] >= k) {
        s_bin = kBins - 1 - 8 * tid - j;
        s_above = above;
      }
      above += v[j];
    }
  }
  __syncthreads();
  const int T = s_bin;  // -1: every visible entry is selected

  // ---- filter this CTA's slice ----
  const int64_t lo = n * blockIdx.x / gridDim.x, hi = n * (blockIdx.x + 1) / gridDim.x;
  const float* sc = a.scores + (size_t)q * a.n_cap;
  uint64_t* sure = a.sure + (size_t)q * k;
  uint64_t* bnd = a.bnd + (size_t)q * a.n_cap;
  for (int64_t base = lo; base < hi; base += blockDim.x) {
    const int64_t i = base + tid;
    const bool in = i < hi;
    const uint32_t key = in ? float_key(sc[i]) : 0u;
    const int bin = (int)(key >> 20);
    const uint64_t v = sel_value(key, (uint32_t)i);
    append(in && bin > T, v, &cnt[0], sure, k);
    append(in && bin == T, v, &cnt[1], bnd, (int)a.n_cap);
  }

  // ---- the last CTA of this query finishes the selection ----
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(&cnt[2], 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int ns = min(*(volatile int*)&cnt[0], k);
  const int nb = min(*(volatile int*)&cnt[1], (int)a.n_cap);
  int kk = nsel - ns;  // still to take from the boundary list
  if (kk < 0) kk = 0;
  if (kk > nb) kk = nb;
  for (int i = tid; i < ns; i += blockDim.x) pairs[i] = ~sure[i];
  if (tid == 0) s_fill = ns;
  __syncthreads();
  if (kk > 0) {
    const bool cached = nb <= kBndCache;
    if (cached)
      for (int i = tid; i < nb; i += blockDim.x) bcache[i] = bnd[i];
    __syncthreads();
    const uint64_t* L = cached ? bcache : bnd;
    uint64_t thr = 0;  // take every boundary value >= thr
    if (kk < nb) {
      // every boundary value shares the top 12 key bits (bin T): start below them
      uint64_t prefix = (uint64_t)T << 52, mask = (uint64_t)0xfff << 52;
      int need = kk;
      for (int hi_bit = 52; hi_bit > 0;) {
        const int width = hi_bit >= 8 ? 8 : hi_bit;
        const int shift = hi_bit - width;
        const uint64_t dmask = ((uint64_t)1 << width) - 1;
        for (int i = tid; i < 256; i += blockDim.x) hist256[i] = 0;
        if (tid == 0) s_fill_exact = 0;
        __syncthreads();
        for (int i = tid; i < nb; i += blockDim.x) {
          const uint64_t v = L[i];
          if ((v & mask) == prefix) atomicAdd(&hist256[(v >> shift) & dmask], 1);
        }
        __syncthreads();
        if (tid < 32) {
          int c[8], s = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            c[j] = hist256[255 - 8 * lane - j];
            s += c[j];
          }
          int incl = s;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
          }
          int above = incl - s;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (above < need && above + c[j] >= need) {
              s_digit = 255 - 8 * lane - j;
              s_dabove = above;
              s_fill_exact = (above + c[j] == need);  // the digit's bucket is taken whole
            }
            above += c[j];
          }
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
    for (int i = tid; i < nb; i += blockDim.x) {
      const uint64_t v = L[i];
      if (v >= thr) {
        const int pos = atomicAdd(&s_fill, 1);
        if (pos < kMaxTopk) pairs[pos] = ~v;
      }
    }
  }
  __syncthreads();
  int P = 1;
  while (P < k) P <<= 1;
  const int filled = min(s_fill, nsel);
  for (int i = filled + tid; i < P; i += blockDim.x) pairs[i] = ~0ull;
  __syncthreads();
  bitonic_sort_u64(pairs, P);
  int32_t* out = a.out_idx + (size_t)q * k;
  for (int i = tid; i < k; i += blockDim.x)
    out[i] = i < filled ? (int32_t)(pairs[i] & 0xffffffffu) : -1;
}

}  // namespace

bool topk_decode_path(int B, int T, int64_t n_cap, int k) {
  return (int64_t)B * T <= 64 && n_cap >= 8192 && k <= kMaxTopk;
}

static size_t rup(size_t x) { return (x + 255) / 256 * 256; }

size_t topk_decode_ws_bytes(int B, int T, int64_t n_cap, int k) {
  const size_t Q = (size_t)B * T;
  return rup(Q * kBins * 4) + rup(Q * 16) + rup(Q * k * 8) + rup(Q * (size_t)n_cap * 8);
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
  a.sure = reinterpret_cast<uint64_t*>(p);
  p += rup(Q * t.k * 8);
  a.bnd = reinterpret_cast<uint64_t*>(p);
  return a;
}

cudaError_t topk_decode_clear(const TopkDecodeArgs& a, cudaStream_t st) {
  // hist and cnt are adjacent at the start of the workspace
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
