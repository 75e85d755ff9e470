// Stage 3: top-k selector.
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): C_t^SprsComp keeps the entries whose index score is
// among the top-k of I[t,:]. The result here is ordered by (score desc, index asc) and
// padded with -1 when fewer than k entries are visible; it depends only on the scores.
//
// Rows of up to 16384 entries (prefill chunks): one CTA of 512 threads per query row loads
// the row's order-preserving 32-bit keys into shared memory once; an MSB-first radix
// select over them (digits of 12, 12 and 8 bits, histograms in shared memory, stopping as
// soon as the k-th key's digit bin is taken whole) finds the threshold T and how many keys
// equal to T are needed. The keys above T and those ties are appended (warp-aggregated,
// any order; ties in index order when only some are taken), and a bitonic sort of the
// (key, index) pairs orders them.
//
// Longer rows: one CTA of 1024 threads per row re-reads the scores from global memory for
// each of 4 radix passes of 8 bits, then appends every entry with key >= T and sorts; only
// when ties at T overflow the 2048 shared slots does a block-wide scan in index order
// gather the keys > T and the first (lowest-index) keys == T instead.
#include "common.cuh"
#include "internal.h"
#include "qhat.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;

__device__ __forceinline__ uint64_t pack_desc(uint32_t key, uint32_t idx) {
  return ((uint64_t)(~key) << 32) | idx;  // ascending order = key desc, index asc
}

// Exclusive block scan of one flag per thread; returns this thread's offset, *total = sum.
__device__ __forceinline__ int block_excl_scan(bool flag, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) wsum[wid] = __popc(bal);
  __syncthreads();
  if (wid == 0) {
    const int v = wsum[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    wsum[32 + lane] = incl - v;
    if (lane == 31) wsum[64] = incl;
  }
  __syncthreads();
  const int off = wsum[32 + wid] + in_warp;
  *total = wsum[64];
  __syncthreads();
  return off;
}

__device__ void bitonic_sort(uint64_t* arr, int P) {
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

template <typename TS>
__global__ void __launch_bounds__(kThreads) k_topk_rows(TopkArgs a) {
  __shared__ uint64_t pairs[kMaxTopk];
  __shared__ int hist[256];
  __shared__ int wsum[72];
  __shared__ uint32_t sel_digit;
  __shared__ int sel_above;
  const int bt = blockIdx.x;
  const int64_t t = a.q_pos[bt];
  if (a.qj.qhat != nullptr) {  // side job: this row's query heads for the attention
    __shared__ float s_cs[256], s_sn[256];
    qhat_rows(a.qj, bt, (double)t, 0, a.qj.H, s_cs, s_sn);
    __syncthreads();
  }
  const int64_t n = t < 0 ? 0 : (t / a.m < a.n_cap ? t / a.m : a.n_cap);
  const TS* sc = (sizeof(TS) == 4 ? static_cast<const TS*>(static_cast<const void*>(a.scores))
                                  : static_cast<const TS*>(a.scores16)) + (size_t)bt * a.n_cap;
  int32_t* out = a.out_idx + (size_t)bt * a.k;
  const int k = a.k;
  int P = 1;
  while (P < k) P <<= 1;

  if (n <= k) {  // everything visible is selected; just order it
    for (int i = threadIdx.x; i < P; i += blockDim.x)
      pairs[i] = i < n ? pack_desc(float_key(ld_score(sc, i)), (uint32_t)i) : ~0ull;
    __syncthreads();
    bitonic_sort(pairs, P);
    for (int i = threadIdx.x; i < k; i += blockDim.x)
      out[i] = i < n ? (int32_t)(pairs[i] & 0xffffffffu) : -1;
    return;
  }

  // radix select of the k-th largest key
  uint32_t prefix = 0, mask = 0;
  int kk = k;  // how many still to take among keys matching `prefix`
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t u = float_key(ld_score(sc, i));
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 0xff], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // find the digit holding the kk-th largest: suffix sums
      const int lane = threadIdx.x;
      int v[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {  // lane owns digits 255-8*lane-j (descending)
        v[j] = hist[255 - 8 * lane - j];
        s += v[j];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      int above = incl - s;  // count of keys in digits above this lane's range
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (above < kk && above + v[j] >= kk) {
          sel_digit = 255 - 8 * lane - j;
          sel_above = above;
        }
        above += v[j];
      }
    }
    __syncthreads();
    prefix |= sel_digit << shift;
    mask |= 0xffu << shift;
    kk -= sel_above;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the k-th largest key; take kk of the keys equal to it
  // Every entry with key >= T, in any order: the sort below orders them by (key desc, index
  // asc), so its first k are the keys > T followed by the kk lowest-index keys == T.
  {
    __shared__ int s_cnt;
    if (threadIdx.x == 0) s_cnt = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int64_t base = 0; base < n; base += blockDim.x) {
      const int64_t i = base + threadIdx.x;
      const uint32_t u = i < n ? float_key(ld_score(sc, i)) : 0u;
      const bool take = i < n && u >= T;
      const unsigned bal = __ballot_sync(0xffffffffu, take);
      if (bal == 0) continue;
      int pos = 0;
      if (lane == __ffs(bal) - 1) pos = atomicAdd(&s_cnt, __popc(bal));
      pos = __shfl_sync(0xffffffffu, pos, __ffs(bal) - 1) + __popc(bal & ((1u << lane) - 1u));
      if (take && pos < kMaxTopk) pairs[pos] = pack_desc(u, (uint32_t)i);
    }
    __syncthreads();
    const int cnt = s_cnt;
    if (cnt <= kMaxTopk) {
      int Pc = 1;
      while (Pc < cnt) Pc <<= 1;
      for (int i = cnt + threadIdx.x; i < Pc; i += blockDim.x) pairs[i] = ~0ull;
      __syncthreads();
      bitonic_sort(pairs, Pc);
      for (int i = threadIdx.x; i < k; i += blockDim.x)
        out[i] = (int32_t)(pairs[i] & 0xffffffffu);
      return;
    }
    __syncthreads();  // too many ties for shared memory: the ordered gather below
  }
  const int n_gt = k - kk;
  int run_gt = 0, run_eq = 0;
  for (int64_t base = 0; base < n; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    const uint32_t u = i < n ? float_key(ld_score(sc, i)) : 0u;
    const bool gt = i < n && u > T, eq = i < n && u == T;
    int tot_gt, tot_eq;
    const int o_gt = block_excl_scan(gt, wsum, &tot_gt);
    const int o_eq = block_excl_scan(eq, wsum, &tot_eq);
    if (gt) pairs[run_gt + o_gt] = pack_desc(u, (uint32_t)i);
    if (eq && run_eq + o_eq < kk) pairs[n_gt + run_eq + o_eq] = pack_desc(u, (uint32_t)i);
    run_gt += tot_gt;
    run_eq += tot_eq;
  }
  for (int i = k + threadIdx.x; i < P; i += blockDim.x) pairs[i] = ~0ull;
  __syncthreads();
  bitonic_sort(pairs, P);
  for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = (int32_t)(pairs[i] & 0xffffffffu);
}


// ---------------------------------------------------------------------------
// rows of up to kRowKeys entries: keys resident in shared memory
// ---------------------------------------------------------------------------
constexpr int kRThreads = 512;
constexpr int kRowKeys = 16384;

// Exclusive scan of one int per thread over the block (512 threads); *total = sum.
__device__ __forceinline__ int block_excl_scan_int(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kRThreads / 32; ++w) {
    const int x = wsum[w];
    base += w < wid ? x : 0;
    tot += x;
  }
  *total = tot;
  __syncthreads();  // wsum may be reused
  return base + incl - v;
}

// The bin of a descending walk over hist[0..nbins) in which the count reaches `need`
// (1 <= need <= sum): *bin, and *above = the count in the bins above it.
__device__ __forceinline__ void find_bin(const int* hist, int nbins, int need, int* wsum,
                                         int* s_bin, int* s_above) {
  const int tid = threadIdx.x;
  const int per = nbins >= kRThreads ? nbins / kRThreads : 1;
  const int first = nbins - 1 - tid * per;  // this thread's bins: first, first-1, ...
  int v[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = (j < per && first - j >= 0) ? hist[first - j] : 0;
    sum += v[j];
  }
  int total;
  int above = block_excl_scan_int(sum, wsum, &total);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < per && first - j >= 0 && above < need && above + v[j] >= need) {
      *s_bin = first - j;
      *s_above = above;
    }
    above += v[j];
  }
  __syncthreads();
}

// Ascending bitonic sort of arr[0..512) with one element per thread (512 threads): partners
// closer than a warp are exchanged by shuffles, farther ones through `buf` (512 entries, one
// barrier per such stage), so only 10 of the 45 stages wait on the block. On return
// arr[i] holds the i-th smallest.
__device__ __forceinline__ void bitonic_sort512(uint64_t* arr, uint64_t* buf) {
  const int tid = threadIdx.x;
  uint64_t x = arr[tid];
  uint64_t* cur = arr;  // exchange buffer of the next cross-warp stage (alternates)
#pragma unroll
  for (int size = 2; size <= 512; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      uint64_t y;
      if (stride >= 32) {
        uint64_t* b = cur;
        cur = cur == arr ? buf : arr;
        __syncthreads();  // the previous readers of b are done
        b[tid] = x;
        __syncthreads();
        y = b[tid ^ stride];
      } else {
        const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)x, stride);
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(x >> 32), stride);
        y = ((uint64_t)hi << 32) | lo;
      }
      const bool asc = (tid & size) == 0, lower = (tid & stride) == 0;
      x = (lower == asc) ? (x < y ? x : y) : (x < y ? y : x);
    }
  }
  __syncthreads();
  arr[tid] = x;
  __syncthreads();
}

template <typename TS>
__global__ void __launch_bounds__(kRThreads, 2) k_topk_rows_smem(TopkArgs a, int vec) {
  extern __shared__ __align__(16) uint32_t kq[];  // the row's keys
  __shared__ __align__(16) uint64_t s_u[kMaxTopk];  // histogram (ints), then (key, index) pairs
  __shared__ uint64_t s_sortbuf[kRThreads];
  __shared__ int wsum[kRThreads / 32];
  __shared__ int s_bin, s_above;
  int* hist = reinterpret_cast<int*>(s_u);
  uint64_t* pairs = s_u;
  const int tid = threadIdx.x;
  const int bt = blockIdx.x;
  const int64_t t = a.q_pos[bt];
  const int n = (int)(t < 0 ? 0 : (t / a.m < a.n_cap ? t / a.m : a.n_cap));
  const TS* sc = (sizeof(TS) == 4 ? static_cast<const TS*>(static_cast<const void*>(a.scores))
                                  : static_cast<const TS*>(a.scores16)) + (size_t)bt * a.n_cap;
  // fp32 rows in groups of 4 straight into shared memory; they land during the side job
  const bool async_row = sizeof(TS) == 4 && vec;
  if (async_row) {
    const int ng = (n + 3) >> 2;
    const uint32_t dst = (uint32_t)__cvta_generic_to_shared(kq);
    for (int g = tid; g < ng; g += kRThreads)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * g),
                   "l"(reinterpret_cast<const float4*>(sc) + g)
                   : "memory");
  }
  if (a.qj.qhat != nullptr) {  // side job: this row's query heads for the attention
    __shared__ float s_cs[256], s_sn[256];
    qhat_rows(a.qj, bt, (double)t, 0, a.qj.H, s_cs, s_sn);
  }
  int32_t* out = a.out_idx + (size_t)bt * a.k;
  const int k = a.k;
  int P = 1;
  while (P < k) P <<= 1;

  // ---- keys into shared memory (groups of 4 by vector loads when rows are 16-byte aligned;
  //      each thread converts the groups it copied) ----
  if (async_row) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    const int ng = (n + 3) >> 2;
    for (int g = tid; g < ng; g += kRThreads) {
      const uint4 x = reinterpret_cast<const uint4*>(kq)[g];
      reinterpret_cast<uint4*>(kq)[g] =
          make_uint4(float_key(__uint_as_float(x.x)), float_key(__uint_as_float(x.y)),
                     float_key(__uint_as_float(x.z)), float_key(__uint_as_float(x.w)));
    }
  } else if (vec) {
    const int ng = (n + 3) >> 2;
#pragma unroll 8
    for (int g = tid; g < ng; g += kRThreads) {
      float f[4];
      if constexpr (sizeof(TS) == 4) {
        const float4 x = reinterpret_cast<const float4*>(sc)[g];
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
      } else {
        const uint2 x = reinterpret_cast<const uint2*>(sc)[g];
        f[0] = __uint_as_float(x.x << 16); f[1] = __uint_as_float(x.x & 0xffff0000u);
        f[2] = __uint_as_float(x.y << 16); f[3] = __uint_as_float(x.y & 0xffff0000u);
      }
      reinterpret_cast<uint4*>(kq)[g] =
          make_uint4(float_key(f[0]), float_key(f[1]), float_key(f[2]), float_key(f[3]));
    }
  } else {
    for (int i = tid; i < n; i += kRThreads) kq[i] = float_key(ld_score(sc, i));
  }
  for (int i = tid; i < 4096; i += kRThreads) hist[i] = 0;
  __syncthreads();

  if (n <= k) {  // everything visible is selected; just order it
    for (int i = tid; i < P; i += kRThreads) pairs[i] = i < n ? pack_desc(kq[i], (uint32_t)i) : ~0ull;
    __syncthreads();
    bitonic_sort(pairs, P);
    for (int i = tid; i < k; i += kRThreads)
      out[i] = i < n ? (int32_t)(pairs[i] & 0xffffffffu) : -1;
    return;
  }

  // ---- radix select of the k-th largest key: digits [31:20], [19:8], [7:0] ----
  int kk = k;          // still to take among keys matching the prefix
  uint32_t T = 0;      // threshold: every key >= T is taken ...
  bool ties = false;   // ... unless only kk of the keys == T are (then in index order)
  {
    for (int i = tid; i < n; i += kRThreads) atomicAdd(&hist[kq[i] >> 20], 1);
    __syncthreads();
    find_bin(hist, 4096, kk, wsum, &s_bin, &s_above);
    const uint32_t b1 = (uint32_t)s_bin;
    kk -= s_above;
    const int in1 = hist[b1];
    __syncthreads();
    if (in1 == kk) {
      T = b1 << 20;
    } else {
      for (int i = tid; i < 4096; i += kRThreads) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kRThreads) {
        const uint32_t u = kq[i];
        if ((u >> 20) == b1) atomicAdd(&hist[(u >> 8) & 0xfffu], 1);
      }
      __syncthreads();
      find_bin(hist, 4096, kk, wsum, &s_bin, &s_above);
      const uint32_t b2 = (b1 << 12) | (uint32_t)s_bin;
      kk -= s_above;
      const int in2 = hist[s_bin];
      __syncthreads();
      if (in2 == kk) {
        T = b2 << 8;
      } else {
        for (int i = tid; i < 256; i += kRThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kRThreads) {
          const uint32_t u = kq[i];
          if ((u >> 8) == b2) atomicAdd(&hist[u & 0xffu], 1);
        }
        __syncthreads();
        find_bin(hist, 256, kk, wsum, &s_bin, &s_above);
        T = (b2 << 8) | (uint32_t)s_bin;
        kk -= s_above;
        ties = hist[s_bin] > kk;
        __syncthreads();
      }
    }
  }

  // ---- append: keys > T (or >= T when the whole tie group is taken), any order: each
  //      thread counts its own, one block scan places them ----
  {
    const uint32_t Tl = ties ? T + 1u : T;  // take u >= Tl
    const bool none = ties && T == 0xffffffffu;  // no key above the largest
    int mine = 0;
    for (int i = tid; i < n && !none; i += kRThreads) mine += kq[i] >= Tl ? 1 : 0;
    int tot;
    int pos = block_excl_scan_int(mine, wsum, &tot);
    for (int i = tid; i < n && mine > 0; i += kRThreads) {
      const uint32_t u = kq[i];
      if (u >= Tl) {
        pairs[pos++] = pack_desc(u, (uint32_t)i);
        --mine;
      }
    }
  }
  if (ties) {  // the first kk keys == T in index order
    const int n_gt = k - kk;
    int run = 0;
    for (int base = 0; base < n && run < kk; base += kRThreads) {
      const int i = base + tid;
      const bool eq = i < n && kq[i] == T;
      int tot;
      const int off = block_excl_scan_int(eq ? 1 : 0, wsum, &tot);
      if (eq && run + off < kk) pairs[n_gt + run + off] = pack_desc(T, (uint32_t)i);
      run += tot;
    }
  }
  if (P <= kRThreads) P = kRThreads;  // one element per thread: the shuffle network
  for (int i = k + tid; i < P; i += kRThreads) pairs[i] = ~0ull;
  __syncthreads();
  if (P == kRThreads) bitonic_sort512(pairs, s_sortbuf);
  else bitonic_sort(pairs, P);
  for (int i = tid; i < k; i += kRThreads) out[i] = (int32_t)(pairs[i] & 0xffffffffu);
}

}  // namespace

size_t topk_workspace_bytes(int B, int T, int64_t n_cap, int k) {
  return topk_decode_path(B, T, n_cap, k) ? topk_decode_ws_bytes(B, T, n_cap, k) : 0;
}

cudaError_t launch_topk(const TopkArgs& a, void* ws, size_t ws_bytes, cudaStream_t st,
                        bool hist_ready) {
  if (a.B == 0 || a.T == 0) return cudaSuccess;
  if (topk_decode_path(a.B, a.T, a.n_cap, a.k)) {
    if (ws == nullptr || ws_bytes < topk_decode_ws_bytes(a.B, a.T, a.n_cap, a.k))
      return cudaErrorInvalidValue;
    return launch_topk_decode(topk_decode_args(a, ws), hist_ready, st);
  }
  const bool b16 = a.scores16 != nullptr;
  if (a.n_cap <= kRowKeys) {
    // vector loads need every row start 16-byte (fp32) or 8-byte (bf16) aligned
    const uintptr_t p = b16 ? (uintptr_t)a.scores16 : (uintptr_t)a.scores;
    const int vec = (a.n_cap % 4 == 0 && p % 16 == 0) ? 1 : 0;
    const size_t smem = (size_t)((a.n_cap + 3) / 4 * 4) * 4;
    auto kern = b16 ? k_topk_rows_smem<__nv_bfloat16> : k_topk_rows_smem<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kRowKeys * 4));
    if (e != cudaSuccess) return e;
    return launch(false, kern, dim3(a.B * a.T), dim3(kRThreads), smem, st, a, vec);
  }
  if (b16)
    return launch(false, k_topk_rows<__nv_bfloat16>, dim3(a.B * a.T), dim3(kThreads), 0, st, a);
  return launch(false, k_topk_rows<float>, dim3(a.B * a.T), dim3(kThreads), 0, st, a);
}

}  // namespace csa
