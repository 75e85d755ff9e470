// Stage 1: token-level KV compression, optionally finalised with RMSNorm + RoPE.
//
// 【论文解读】DeepSeek-V4, 一(三)1(1) 压缩 KV Entries: entry i of a CSA layer is a
// per-channel softmax-weighted sum over 2m tokens -- the a-branch of block i and the
// b-branch of block i-1 -- with learned positional biases B^a, B^b; block 0 pads the
// b-branch with -inf logits and zero values. 一(三)2(1) (HCA): one branch over the m'
// tokens of block i. 一(三)3(1)/(2): the entry head is RMSNorm'd and its last r dims
// rotated (position m*i) before attention.
//
// Layout: one CTA per (entry, request); each thread owns channel pairs. The pooled row is
// kept in shared memory for the RMS reduction and the RoPE pairs. HBM-bound: every input
// element is read once (2m*4 values per channel), coalesced across the channel axis.
#include "common.cuh"
#include "internal.h"

namespace csa {

__device__ int g_compress_error = 0;  // 331: a page id outside the pool (the entry is skipped)

template <typename T, bool kPaged>
__device__ __forceinline__ void compress_body(const CompressArgs& a, const CompressPages& pg) {
  extern __shared__ float row[];  // [c]
  __shared__ float red[32];
  const int i = blockIdx.x;       // entry within the chunk
  const int b = blockIdx.y;       // request
  const int c = a.c, m = a.m;
  const T* Ca = static_cast<const T*>(a.Ca) + (size_t)b * a.n_tok * c;
  const T* Za = static_cast<const T*>(a.Za) + (size_t)b * a.n_tok * c;
  const T* Cb = a.Cb ? static_cast<const T*>(a.Cb) + (size_t)b * a.n_tok * c : nullptr;
  const T* Zb = a.Zb ? static_cast<const T*>(a.Zb) + (size_t)b * a.n_tok * c : nullptr;
  const T* pCb = a.prev_Cb ? static_cast<const T*>(a.prev_Cb) + (size_t)b * m * c : nullptr;
  const T* pZb = a.prev_Zb ? static_cast<const T*>(a.prev_Zb) + (size_t)b * m * c : nullptr;
  const T* bias = static_cast<const T*>(a.bias);

  // b-branch source: block i-1 of this chunk, the previous chunk's tail, or nothing
  const T* srcCb = nullptr;
  const T* srcZb = nullptr;
  if (a.overlap) {
    if (i > 0) {
      srcCb = Cb + (size_t)m * (i - 1) * c;
      srcZb = Zb + (size_t)m * (i - 1) * c;
    } else if (pCb) {
      srcCb = pCb;
      srcZb = pZb;
    }
  }
  float ss = 0.f;
  for (int j = threadIdx.x; j < c; j += blockDim.x) {
    // pass 1: max of the logits of this channel
    float mx = -INFINITY;
    for (int r = 0; r < m; ++r)
      mx = fmaxf(mx, to_f32(Za[((size_t)m * i + r) * c + j]) + to_f32(bias[r * c + j]));
    if (srcZb)
      for (int r = 0; r < m; ++r)
        mx = fmaxf(mx, to_f32(srcZb[(size_t)r * c + j]) + to_f32(bias[(m + r) * c + j]));
    // pass 2: weights and weighted sum
    float den = 0.f, num = 0.f;
    for (int r = 0; r < m; ++r) {
      const float e = expf(to_f32(Za[((size_t)m * i + r) * c + j]) + to_f32(bias[r * c + j]) - mx);
      den += e;
      num = fmaf(e, to_f32(Ca[((size_t)m * i + r) * c + j]), num);
    }
    if (srcZb)
      for (int r = 0; r < m; ++r) {
        const float e =
            expf(to_f32(srcZb[(size_t)r * c + j]) + to_f32(bias[(m + r) * c + j]) - mx);
        den += e;
        num = fmaf(e, to_f32(srcCb[(size_t)r * c + j]), num);
      }
    const float v = num / den;
    row[j] = v;
    ss = fmaf(v, v, ss);
  }
  T* out;
  if constexpr (kPaged) {  // the state cache's page pool
    const int64_t e = a.first_entry + i;
    const int32_t page = pg.page_table[(size_t)b * pg.max_pages + e / pg.page_rows];
    if (page < 0 || page >= pg.n_pages) {  // uniform over the CTA
      if (threadIdx.x == 0) atomicCAS(&g_compress_error, 0, 331);
      return;
    }
    out = static_cast<T*>(a.out) + ((size_t)page * pg.page_rows + (size_t)(e % pg.page_rows)) * c;
  } else {
    out = static_cast<T*>(a.out) + ((size_t)b * a.n_cap + a.first_entry + i) * c;
  }
  if (!a.finalize) {
    __syncthreads();
    for (int j = threadIdx.x; j < c; j += blockDim.x) out[j] = from_f32<T>(row[j]);
    return;
  }
  const float tot = block_sum(ss, red);  // includes a __syncthreads after row[] writes
  const float rstd = rsqrtf(tot / (float)c + a.eps);
  const T* g = static_cast<const T*>(a.rms_w);
  const int r = a.rope_dims, r0 = c - r;
  const double pos = (double)a.m * (double)(a.first_entry + i);
  for (int j = threadIdx.x; j < c; j += blockDim.x) {
    float v = row[j] * rstd * (g ? to_f32(g[j]) : 1.f);
    if (j >= r0) {
      const int p = (j - r0) >> 1;
      const int partner = j ^ 1;  // r0 is even, so pairs are (even, odd)
      const float u = row[partner] * rstd * (g ? to_f32(g[partner]) : 1.f);
      float cs, sn;
      rope_cos_sin(pos, p, r, (double)a.rope_base, &cs, &sn);
      v = ((j - r0) & 1) == 0 ? v * cs - u * sn : u * sn + v * cs;
    }
    out[j] = from_f32<T>(v);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_compress(CompressArgs a) {
  compress_body<T, false>(a, CompressPages{});
}

template <typename T>
__global__ void __launch_bounds__(256) k_compress_paged(CompressArgs a, CompressPages pg) {
  compress_body<T, true>(a, pg);
}

cudaError_t launch_compress(const CompressArgs& a, bool bf16, cudaStream_t st,
                            const CompressPages* pages) {
  const int n_ent = (int)(a.n_tok / a.m);
  if (n_ent == 0 || a.B == 0) return cudaSuccess;
  dim3 grid(n_ent, a.B);
  const int threads = a.c >= 256 ? 256 : ((a.c + 31) / 32) * 32;
  const size_t smem = (size_t)a.c * sizeof(float);
  if (pages != nullptr) {
    if (bf16)
      launch(false, k_compress_paged<__nv_bfloat16>, dim3(grid), dim3(threads), smem, st, a,
             *pages);
    else
      launch(false, k_compress_paged<float>, dim3(grid), dim3(threads), smem, st, a, *pages);
  } else if (bf16) {
    launch(false, k_compress<__nv_bfloat16>, dim3(grid), dim3(threads), smem, st, a);
  } else {
    launch(false, k_compress<float>, dim3(grid), dim3(threads), smem, st, a);
  }
  return cudaGetLastError();
}

cudaError_t compress_device_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_compress_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_compress_error, &zero, sizeof(int));
}

}  // namespace csa
