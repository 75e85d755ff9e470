// Stage 3: top-k selector.
//
// 【论文解读】DeepSeek-V4, 一(三)1(2): C_t^SprsComp keeps the entries whose index score is
// among the top-k of I[t,:]. The result here is ordered by (score desc, index asc) and
// padded with -1 when fewer than k entries are visible; it depends only on the scores.
//
// One CTA of 1024 threads per query row: an MSB-first radix select on order-preserving
// 32-bit keys (4 passes of 8 bits, histograms in shared memory) finds the k-th largest
// key T. Every entry with key >= T is then appended (warp-aggregated, any order) and a
// bitonic sort of the (key, index) pairs orders them; its first k are the result. Only
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
  if (a.scores16 != nullptr)
    return launch(false, k_topk_rows<__nv_bfloat16>, dim3(a.B * a.T), dim3(kThreads), 0, st, a);
  return launch(false, k_topk_rows<float>, dim3(a.B * a.T), dim3(kThreads), 0, st, a);
}

}  // namespace csa
