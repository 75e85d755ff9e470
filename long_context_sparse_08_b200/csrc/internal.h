// Internal launch interface of libcsa: argument blocks passed by value to the kernels and
// the launchers the C ABI layer (api.cu) calls after validating its arguments.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace csa {

// Launch `kernel`; with `pdl` it may start before its predecessor in the stream ends (the
// kernel calls pdl_wait() before it reads what a predecessor wrote).
void count_launch();  // every kernel launch of the library goes through launch()
template <typename... KArgs, typename... Args>
cudaError_t launch(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t st, Args... args) {
  count_launch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

struct CompressArgs {
  int B, m, c, overlap, rope_dims, finalize;
  int64_t n_tok, first_entry, n_cap;
  float rope_base, eps;
  const void *Ca, *Cb, *Za, *Zb, *bias, *prev_Cb, *prev_Zb, *rms_w;
  void* out;
};
// Page pool of a paged compression: entry e of request b goes to row e % page_rows of page
// page_table[b * max_pages + e / page_rows] of `out`.
struct CompressPages {
  const int32_t* page_table;
  int page_rows, max_pages, n_pages;
};
// pages == nullptr: the contiguous cache [B, n_cap, c]
cudaError_t launch_compress(const CompressArgs& a, bool bf16, cudaStream_t st,
                            const CompressPages* pages = nullptr);

namespace proj { struct Geom; }
struct OutProjArgs;
// grouped output projection (decode: Q <= 16 queries)
proj::Geom out_proj_geom(int Q, int H, int c, int g, int d_g, int d);
size_t out_proj_workspace_bytes(const proj::Geom& G);
cudaError_t launch_out_proj(OutProjArgs a, void* ws, cudaStream_t st);
// prefill form on tensor cores (Q >= 128 queries)
bool out_proj_tc_shape_ok(const proj::Geom& G);
size_t out_proj_tc_workspace_bytes(const proj::Geom& G);
cudaError_t launch_out_proj_tc(const OutProjArgs& a, void* ws, cudaStream_t st);
cudaError_t out_proj_tc_device_error(int* code);

namespace state { struct Args; }
// decode-time append of one token per request into the state cache and its pages
cudaError_t launch_state_append(const state::Args& a, bool bf16, cudaStream_t st);
// rows [B, n, c] (io dtype) = entries first_entry .. first_entry + n - 1 into their pages in
// the format a.out (csa_encode_paged)
cudaError_t launch_encode_paged(const state::Args& a, bool bf16, const void* rows, int64_t n,
                                int64_t first_entry, cudaStream_t st);
cudaError_t state_append_device_error(int* code);
// after a prefill chunk: its last raw rows and window rows into the state cache
cudaError_t launch_state_resume(const state::Args& a, bool bf16, int64_t first_tok,
                                int64_t n_tok, cudaStream_t st);
cudaError_t compress_device_error(int* code);

struct IndexArgs {
  int B, T, m, n_idx_heads, d_idx, kdt;
  int64_t n_cap;
  const void *qI, *qI_scale, *KI, *KI_scale;
  const float* w;
  const int64_t* q_pos;
  float* scores;  // [B, T, n_cap]
  int* hist;      // optional [B*T][4096] histogram of the scores' top 12 key bits (zeroed)
  void* scores16;  // non-null: the scores are rounded to bf16 and stored here instead
  const int32_t* page_table;  // non-null: KI / KI_scale are a pool of n_pages pages of
                              // page_rows keys; key e of request b is row e % page_rows of
                              // page page_table[b * max_pages + e / page_rows]
  int page_rows, max_pages, n_pages;
};
// *hist_done: whether the launched kernel also filled a.hist
cudaError_t launch_index_scores(const IndexArgs& a, cudaStream_t st, bool* hist_done = nullptr);
// tensor-core kernel for MXFP4 keys (64 heads x 128 dims, N_cap % 32 == 0)
bool index_mxf4_tc_supported(const IndexArgs& a);
cudaError_t launch_index_mxf4_tc(const IndexArgs& a, cudaStream_t st);
cudaError_t index_mxf4_device_error(int* code);
// tensor-core kernel for FP8 (e4m3 + row scale) and bf16 keys with bf16 queries (64 heads x
// 128 dims, N_cap % 128 == 0; launched over batches of at most 512 queries)
bool index_bf16_tc_supported(const IndexArgs& a);
cudaError_t launch_index_bf16_tc(const IndexArgs& a, cudaStream_t st);
cudaError_t index_bf16_device_error(int* code);

// q_hat = RoPE_t(RMSNorm(q) * q_rms_w) in bf16 for the attention that follows a top-k: an
// optional side job of the decode selector (c = 512, bf16 io)
struct QhatJob {
  const void* q;        // bf16 [B*T][H][c]
  const void* q_rms_w;  // bf16 [c] or nullptr
  void* qhat;           // bf16 [B*T][H][c]; nullptr: no job
  int H, r;
  float eps, rope_base;
  double inv_freq[64];  // RoPE pair frequencies, formed on the host (r <= 128)
};

struct TopkArgs {
  int B, T, m, k;
  int64_t n_cap;
  const float* scores;
  const void* scores16;  // non-null: bf16 scores [B, T, n_cap] in place of `scores`
  const int64_t* q_pos;
  int32_t* out_idx;
  QhatJob qj;
};
size_t topk_workspace_bytes(int B, int T, int64_t n_cap, int k);
cudaError_t launch_topk(const TopkArgs& a, void* ws, size_t ws_bytes, cudaStream_t st,
                        bool hist_ready = false);

// few long rows (decode): histogram + filter + last-CTA selection
struct TopkDecodeArgs {
  int Q, m, k, nslice;
  int64_t n_cap;
  const float* scores;
  const void* scores16;  // non-null: bf16 scores in place of `scores`
  const int64_t* q_pos;
  int32_t* out_idx;
  int* hist;          // [Q][4096]
  int* cnt;           // [Q][4]: sure count, boundary count, ticket
  uint64_t* list;     // [Q][k + n_cap]: sure list (k), then boundary list (n_cap)
  QhatJob qj;
};
bool topk_decode_path(int B, int T, int64_t n_cap, int k);
size_t topk_decode_ws_bytes(int B, int T, int64_t n_cap, int k);
TopkDecodeArgs topk_decode_args(const TopkArgs& t, void* ws);
cudaError_t topk_decode_clear(const TopkDecodeArgs& a, cudaStream_t st);
cudaError_t launch_topk_decode(TopkDecodeArgs a, bool hist_ready, cudaStream_t st);

struct MqaArgs {
  int B, T, m, H, c, rope_dims, n_win, k;  // k = 0: dense (all visible entries)
  int64_t n_cap, l_raw;
  float rope_base, eps, scale;
  const void *q, *kv, *win, *q_rms_w;
  const int32_t* idx;
  const int64_t *q_pos, *win_pos0;
  const float* sink;
  void* out;
  bool chained;  // the previous launch on the stream is a kernel of this library that has
                 // waited for its own predecessors (the attention may then prepare its
                 // queries before its own wait)
  const void* qhat;  // bf16 [B*T][H][c] prepared q_hat (written by an earlier kernel of the
                     // chain) or nullptr: the attention prepares it
  const float* kv_scale;  // non-null: `kv` holds mixed-precision rows (c - r e4m3 codes, then
                          // r bf16 values; c + r bytes) and this their per-row scales
  const int32_t* page_table;  // non-null: `kv` (and kv_scale) are a pool of n_pages pages of
                              // page_rows rows; entry e of request b is row e % page_rows of
                              // page page_table[b * max_pages + e / page_rows];
                              // n_cap = page_rows * max_pages
  int page_rows, max_pages, n_pages;
};
size_t mqa_workspace_bytes(const MqaArgs& a);
// tensor-core attention (bf16, c = 512, heads in groups of 64)
bool mqa_tc_supported(const MqaArgs& a, bool bf16);
size_t mqa_tc_workspace_bytes(const MqaArgs& a);
// zero two 16-byte aligned ranges (sizes multiples of 16; the second may be empty) in
// stream order; programmatic launch, waits for its predecessors
cudaError_t launch_zero(void* p0, size_t b0, void* p1, size_t b1, cudaStream_t st);
cudaError_t launch_mqa_tc(const MqaArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);
cudaError_t mqa_tc_device_error(int* code);
cudaError_t launch_mqa(const MqaArgs& a, bool bf16, void* ws, size_t ws_bytes, cudaStream_t st);

// Records a formatted message as the calling thread's csa_last_error() and returns `s`.
csa_status report_error(csa_status s, const char* fmt, ...);

// benchmarking hook (see csa_set_index_timing_events)
void timing_before(cudaStream_t st);
void timing_after(cudaStream_t st);

}  // namespace csa
