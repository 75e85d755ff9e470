/*
 * csa.h -- C ABI of the CSA / HCA attention hot path (DeepSeek-V4 hybrid attention)
 * for one NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [P1] 【论文解读】DeepSeek-V4, 一、模型架构 (三) 混合注意力架构：CSA + HCA:
 *        1(1) 压缩 KV Entries (overlapped compression), 1(2) Lightning Indexer 稀疏选择
 *        (index score, visibility, top-k), 1(3) Shared Key-Value MQA, 2(1)/2(2) HCA,
 *        3(1) query / KV RMSNorm, 3(2) partial RoPE and output rotation at -t,
 *        3(3) sliding window, 3(4) attention sink.
 *   [P1'] same page, 二、基础设施 (四) FP4 量化感知训练: the indexer's QK path in FP4.
 *   [P1''] same page, 二、基础设施 (六) 推理框架: state cache and paged cache at inference.
 *   [P4] DeepseekV4论文解析, 2. Hybrid Attention：CSA + HCA (从注意力公式到可部署系统): the
 *        per-request state and the paged cache in logical blocks of lcm(4, 128) = 128 raw
 *        tokens (32 CSA entries or 1 HCA entry).
 *
 * Conventions shared by every call
 *   - Every tensor pointer is device memory owned by the caller; the library never
 *     allocates or frees device memory (the state cache's page allocator owns host memory
 *     only). Scratch comes from a caller-provided workspace whose size
 *     csa_workspace_size() returns.
 *   - Layouts are dense row-major with the shapes given per argument. Pointers must be
 *     16-byte aligned; c is a multiple of 64 (or exactly 64 for fp32 inputs), 0 <= r <= c,
 *     r even.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and return once the kernels are queued. No host synchronisation happens.
 *   - Arguments are validated on the host before any launch; on error nothing is
 *     launched and a status is returned (csa_last_error() gives a one-line reason for
 *     the calling thread). CSA_ERR_CUDA reports a launch failure seen by
 *     cudaGetLastError() right after queueing.
 *   - On the device, top-k indices equal to -1 (or outside [0, N_cap)) are skipped.
 *     Nothing traps.
 *   - Positions (q_pos, win_pos0) are int64 device arrays. A query at position t sees the
 *     compressed entries s < min(floor(t/m), N_cap) ([P1] 1(2)) and the window tokens
 *     max(t-n_win+1, 0) .. t, its own token included ([P1] 3(3)); the window buffer of
 *     request b holds token win_pos0[b]+j in row j and must cover those positions.
 *   - RoPE ([P1] 3(2)): the last r dims, adjacent pairs (2p, 2p+1) of that slice turned by
 *     pos * rope_base^(-2p/r); compressed entry i sits at position m*i. RMSNorm ([P1] 3(1)):
 *     x / sqrt(mean(x^2) + rms_eps) * gamma (gamma = 1 when the weight pointer is NULL).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1, /* a pointer, size or alignment the call cannot accept */
  CSA_ERR_UNSUPPORTED = 2, /* a valid shape / dtype combination this library does not implement */
  CSA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than csa_workspace_size() */
  CSA_ERR_CUDA = 4,        /* the CUDA runtime reported an error while queueing */
  CSA_ERR_NO_PAGES = 5     /* a page pool has too few free pages for the request */
} csa_status;

typedef enum {
  CSA_F32 = 0,               /* IEEE binary32 */
  CSA_BF16 = 1,              /* bfloat16 */
  CSA_FP8_E4M3_ROWSCALE = 2, /* OCP e4m3 codes, one fp32 scale per row (value = code * scale) */
  CSA_MXFP4 = 3,             /* OCP MXFP4: e2m1 pairs per byte (element 2j in the low nibble)
                                and one e8m0 scale byte per 32 elements */
  CSA_MIXED_FP8_BF16 = 4     /* KV entry row ([P1] 一(三)4 item 1): the first c-r values as e4m3
                                codes with one fp32 scale per row (amax of those values / 448),
                                then the last r (RoPE) values as bf16: c + r bytes per row */
} csa_dtype;

/* Method constants, passed by pointer, read on the host during the call only. */
typedef struct {
  int32_t m;           /* tokens per compressed entry: 4 (CSA) or m' = 128 (HCA)        */
  int32_t overlap;     /* 1: CSA a/b overlapped compression; 0: HCA single branch        */
  int32_t c;           /* head dim of queries and compressed KV rows (512 in the models) */
  int32_t rope_dims;   /* r: RoPE on the last r dims (64)                                */
  float rope_base;     /* 10000                                                          */
  float rms_eps;       /* 1e-6                                                           */
  float sm_scale;      /* logit scale; <= 0 means 1/sqrt(c)                              */
  int32_t n_heads;     /* attention query heads H (64 Flash / 128 Pro)                   */
  int32_t n_idx_heads; /* indexer heads H_I (64)                                         */
  int32_t d_idx;       /* indexer head dim d_I (128)                                     */
  int32_t topk;        /* k (512 Flash / 1024 Pro), at most 2048                         */
  int32_t n_win;       /* sliding window n_win (128)                                     */
} csa_params;

/* Which call a workspace is sized for (csa_workspace_size's `entry`). */
typedef enum {
  CSA_WS_INDEX_TOPK = 1,
  CSA_WS_TOPK = 2,
  CSA_WS_SPARSE_MQA = 3,
  CSA_WS_HCA_MQA = 4,
  CSA_WS_FORWARD = 5,
  CSA_WS_INDEX_TOPK_BF16 = 6
} csa_ws_entry;

/*
 * Stage 1 -- token-level KV compression ([P1] 1(1) overlapped; 2(1) non-overlapped),
 * optionally finalised with RMSNorm and RoPE at position m*i ([P1] 3(1), 3(2)).
 *
 * For each request b and new entry i < n_tok/m, channel j:
 *   CSA: softmax over the 2m logits Za[b, m*i+r, j] + bias[r, j] and
 *        Zb[b, m*(i-1)+r, j] + bias[m+r, j] (r < m), weighted sum of Ca / Cb at the same
 *        tokens. For i = 0 the b-branch reads prev_Cb / prev_Zb [B, m, c] (the last m
 *        tokens before this chunk); if those are NULL the chunk starts the sequence and the
 *        b-logits are -inf (values 0).
 *   HCA (overlap = 0): softmax over the m logits Za[b, m*i+r, j] + bias[r, j], weighted sum
 *        of Ca; Cb, Zb, prev_* must be NULL.
 * The entry is written to out_cache[b, first_entry + i, :] ([B, n_cap, c]); with
 * finalize = 1 it is RMSNorm'd (weight kv_rms_w [c] or NULL) and rotated at position
 * m*(first_entry + i). n_tok must be a multiple of m and first_entry + n_tok/m <= n_cap.
 * io: CSA_F32 or CSA_BF16 for every tensor (math is fp32). Ca/Cb/Za/Zb: [B, n_tok, c];
 * bias: [2m, c] (CSA) or [m, c] (HCA).
 */
csa_status csa_compress(const csa_params* p, csa_dtype io, int32_t B, int64_t n_tok,
                        int64_t first_entry, int64_t n_cap, const void* Ca, const void* Cb,
                        const void* Za, const void* Zb, const void* bias, const void* prev_Cb,
                        const void* prev_Zb, const void* kv_rms_w, int32_t finalize,
                        void* out_cache, void* stream);

/*
 * Decode-time compression with a state cache ([P1''] 二、基础设施 (六) 推理框架: a state
 * cache holds the sliding window and the raw tail tokens of an unfinished compression
 * block; finished entries live in a paged cache whose blocks cover a multiple of
 * lcm(m, m') raw tokens -- 128 tokens = 32 CSA entries = 1 HCA entry).
 *
 * Appends one token to each of B requests. For request b, at position t = pos[b]:
 *   - its raw rows go to slot t % S of `state` [B, S, R, c] (io dtype):
 *       CSA (overlap = 1): S = 2m, R = 4 rows in the order Ca, Za, Cb, Zb;
 *       HCA (overlap = 0): S = m,  R = 2 rows in the order C (= Ca), Z (= Za);
 *     the token rows are Ca, Cb, Za, Zb [B, c] (Cb, Zb NULL for HCA);
 *   - win_row [B, c] (final form: normed and rotated by the caller) goes to row t % n_win of
 *     win_ring [B, n_win, c]; both NULL to keep no window;
 *   - when t + 1 is a multiple of m, entry i = t / m is compressed from the state exactly as
 *     csa_compress computes it ([P1] 1(1) / 2(1); the CSA b-branch is block i-1's rows for
 *     i > 0 and absent for i = 0), and with finalize = 1 RMSNorm'd (kv_rms_w [c] or NULL)
 *     and rotated at position m*i ([P1] 3(1), 3(2)). The row goes to row i % page_rows of
 *     page page_table[b, i / page_rows] of `pages`, stored as out_fmt:
 *       out_fmt = io: pages [n_pages, page_rows, c] in the io dtype; page_scales unused;
 *       CSA_FP8_E4M3_ROWSCALE: pages [n_pages, page_rows, c] e4m3 codes (round to nearest
 *         even, saturating), page_scales [n_pages, page_rows] fp32 = amax(row) / 448;
 *       CSA_MXFP4 (c = 128, page_rows a multiple of 128; the indexer keys of [P1'] as
 *         csa_index_scores reads them): pages [n_pages, page_rows, 64] e2m1 pairs (element
 *         2j in the low nibble), page_scales [n_pages, page_rows, 4] e8m0 exponents
 *         floor(log2 amax) - 2 of each 32 values, per block of 128 rows with byte
 *         16*i + 4*j + b holding exponent b of row 32*j + i;
 *       CSA_MIXED_FP8_BF16 (0 < r < c): pages [n_pages, page_rows, c + r] bytes, each row the
 *         e4m3 codes of its first c-r values then its last r values as bf16; page_scales
 *         [n_pages, page_rows] fp32 = amax(first c-r values) / 448.
 *     Indexer keys are compressed like KV entries but take no RMSNorm / RoPE (finalize = 0).
 * The slots of block i-1 and block i are read back, so a request's appends must arrive in
 * position order (one per call), after its state was filled up to t-1: by earlier appends,
 * or, for a request resumed after a prefill, by the caller writing those raw rows into their
 * slots. Requests whose entry's logical page is >= max_pages, whose page id is outside
 * [0, n_pages), or whose position is negative are skipped and leave a device error code
 * (321 position, 322 page slot, 323 page id) for csa_device_error(). The pages use
 * page_rows = 128 / m (a multiple of it for MXFP4 keys); with page_table[b, k] =
 * b * max_pages + k they are the contiguous cache [B, N_cap = page_rows * max_pages, ...]
 * that the attention and indexer calls read.
 * io: CSA_F32 or CSA_BF16 for every input and state tensor (math is fp32); c <= 4096;
 * bias: [2m, c] or [m, c].
 */
csa_status csa_state_append(const csa_params* p, csa_dtype io, int32_t B, const int64_t* pos,
                            const void* Ca, const void* Cb, const void* Za, const void* Zb,
                            const void* win_row, const void* bias, const void* kv_rms_w,
                            int32_t finalize, void* state, void* win_ring, csa_dtype out_fmt,
                            void* pages, void* page_scales, int32_t n_pages, int32_t page_rows,
                            const int32_t* page_table, int32_t max_pages, void* stream);

/*
 * Stage 2 -- lightning-indexer scores ([P1] 1(2)):
 *   I[b,t,s] = sum_h w[b,t,h] * ReLU(qI[b,t,h,:] . KI[b,s,:]),  s < n_vis(b,t),
 * written to out_scores [B, T, N_cap] fp32. Values at s >= n_vis are left unwritten.
 * kdt selects the key format and with it the query format:
 *   CSA_F32:  qI f32 [B,T,H_I,d_I],  KI f32 [B,N_cap,d_I]
 *   CSA_BF16: qI bf16,               KI bf16
 *   CSA_FP8_E4M3_ROWSCALE: qI bf16,  KI e4m3 codes [B,N_cap,d_I] + KI_scale f32 [B,N_cap]
 *   CSA_MXFP4 ([P1'] FP4 QK path): qI [B,T,H_I,d_I/2] bytes + qI_scale [B,T,H_I,d_I/32]
 *             (e8m0, in head order), KI [B,N_cap,d_I/2] bytes + KI_scale [B,N_cap,4] e8m0
 *             stored per block of 128 keys as the tensor cores read it: byte 16*i + 4*j + b
 *             of a block is block-scale b of key 32*j + i. Requires H_I = 64, d_I = 128,
 *             N_cap a multiple of 128 and B*T <= 1024.
 * w: f32 [B,T,H_I]. q_pos: int64 [B,T]. Scores are fp32 sums of exact products.
 * With H_I = 64, d_I = 128 and N_cap a multiple of 128, bf16 and FP8 keys also run on the
 * tensor cores (an e4m3 code widens exactly to bf16; the row scale is applied after the
 * ReLU, which it commutes with as it is positive); other shapes and f32 run on CUDA cores.
 */
csa_status csa_index_scores(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                            int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                            const void* KI, const void* KI_scale, const int64_t* q_pos,
                            float* out_scores, void* stream);

/*
 * Stage 3 -- top-k selector ([P1] 1(2), C_t^SprsComp): for every (b,t), the indices of the
 * k largest scores[b,t,s] over s < n_vis(b,t), ordered by (score descending, index
 * ascending); slots past n_vis hold -1. scores: f32 [B,T,N_cap]; out_idx: int32 [B,T,k].
 * Deterministic: the result depends only on the scores. -0.0 counts as +0.0.
 */
csa_status csa_topk(const csa_params* p, int32_t B, int32_t T, int64_t N_cap,
                    const float* scores, const int64_t* q_pos, int32_t* out_idx, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * Stage 3 as csa_topk, for callers that cannot hand the library device scratch (a host
 * program without a device allocator of its own, or one whose device memory is already
 * reserved for its caches). The paper has no counterpart: this is an interface variant.
 * Allocates nothing: the scratch is one library-owned device array of
 * CSA_TOPK_NOALLOC_SCRATCH_BYTES per device. The first call on a device looks up that
 * array's address (with the device current) and should come before any stream capture.
 * All calls on a device share the array; each call zeroes the counters it needs on its own
 * stream, so calls whose execution overlaps (other streams, other host threads) race:
 * serialise them. Returns CSA_ERR_WORKSPACE, launching nothing, when the call would need
 * more scratch than the array holds (csa_workspace_size(p, CSA_WS_TOPK, ...) bytes; e.g.
 * 4 rows of N_cap = 262144 with k = 1024 need about 8.5 MB; B*T > 64 or N_cap < 8192
 * need none). Results are identical to csa_topk's. Other arguments and errors as csa_topk.
 */
#define CSA_TOPK_NOALLOC_SCRATCH_BYTES (16u << 20)
csa_status csa_topk_noalloc(const csa_params* p, int32_t B, int32_t T, int64_t N_cap,
                            const float* scores, const int64_t* q_pos, int32_t* out_idx,
                            void* stream);

/* Stages 2 + 3 in one call. out_scores may be NULL (the scores then live in the workspace). */
csa_status csa_index_topk(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                          int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                          const void* KI, const void* KI_scale, const int64_t* q_pos,
                          int32_t* out_idx, float* out_scores, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * Stages 2 + 3 with BF16 index scores ([P1'] 二(四): the scores are quantised from FP32 to
 * BF16 before the top-k selector). Each score is computed in fp32 as in csa_index_scores,
 * rounded to the nearest bf16 (ties to even) and stored as bf16 [B, T, N_cap] (out_scores16,
 * or the workspace when NULL); the selector then orders the bf16 values by (value desc,
 * index asc), so scores that round alike tie and the smaller index wins. Half the score
 * bytes of csa_index_topk. Keys: CSA_FP8_E4M3_ROWSCALE, CSA_BF16 or CSA_MXFP4 on the
 * tensor-core indexers (64 heads of 128, N_cap a multiple of 128), else
 * CSA_ERR_UNSUPPORTED. Workspace: csa_workspace_size(..., CSA_WS_INDEX_TOPK_BF16, ...).
 */
csa_status csa_index_topk_bf16(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                               int64_t N_cap, const void* qI, const void* qI_scale,
                               const float* w, const void* KI, const void* KI_scale,
                               const int64_t* q_pos, int32_t* out_idx, void* out_scores16,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 4 -- shared-KV MQA over the selected entries plus the window ([P1] 1(3), 3(1)-(4)).
 * For every (b, t, h): q_hat = RoPE_t(RMSNorm(q[b,t,h,:]) * q_rms_w); the KV rows are
 * kv_cache[b, idx[b,t,j], :] for every valid j followed by the window rows; key = value;
 *   o = sum_j e^{z_j} row_j / (sum_j e^{z_j} + e^{sink[h]}),  z_j = sm_scale * q_hat . row_j,
 * then out[b,t,h,:] = RoPE_{-t}(o). sink may be NULL (no sink). io: CSA_F32 or CSA_BF16 for
 * q [B,T,H,c], kv_cache [B,N_cap,c], win_kv [B,L_raw,c] and out [B,T,H,c]; q_rms_w [c] or
 * NULL (same dtype as io). idx: int32 [B,T,k].
 */
csa_status csa_sparse_mqa(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                          const void* q, const int64_t* q_pos, const void* kv_cache,
                          int64_t N_cap, const int32_t* idx, const void* win_kv, int64_t L_raw,
                          const int64_t* win_pos0, const float* sink, const void* q_rms_w,
                          void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * HCA core attention ([P1] 2(2), 3(1)-(4)): as csa_sparse_mqa, with the KV rows being every
 * visible entry s < min(floor(t/m), N_cap) (m = p->m, e.g. 128) followed by the window.
 */
csa_status hca_dense_mqa(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                         const void* q, const int64_t* q_pos, const void* kv_cache,
                         int64_t N_cap, const void* win_kv, int64_t L_raw,
                         const int64_t* win_pos0, const float* sink, const void* q_rms_w,
                         void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 4 over a mixed-precision KV cache ([P1] 一(三)4 item 1: the RoPE dims in BF16, the
 * rest in FP8): as csa_sparse_mqa / hca_dense_mqa with io = CSA_BF16, except that
 * kv_rows [B, N_cap, c + r] bytes holds each cache row as CSA_MIXED_FP8_BF16 (the e4m3
 * codes of its first c - r values, then its last r values as bf16) and kv_scale
 * [B, N_cap] fp32 the rows' FP8 scales (value = code * scale), as csa_state_append writes
 * them. Window rows stay bf16. The attention widens code * scale to bf16 (one rounding) and
 * then runs as in the bf16 path. Needs c = 512, n_heads a multiple of 64 and rope_dims a
 * multiple of 16 in (0, 512), else CSA_ERR_UNSUPPORTED. Workspace: as the bf16 calls.
 */
csa_status csa_sparse_mqa_mixed_kv(const csa_params* p, int32_t B, int32_t T, const void* q,
                                   const int64_t* q_pos, const void* kv_rows,
                                   const float* kv_scale, int64_t N_cap, const int32_t* idx,
                                   const void* win_kv, int64_t L_raw, const int64_t* win_pos0,
                                   const float* sink, const void* q_rms_w, void* out, void* ws,
                                   size_t ws_bytes, void* stream);
csa_status hca_dense_mqa_mixed_kv(const csa_params* p, int32_t B, int32_t T, const void* q,
                                  const int64_t* q_pos, const void* kv_rows,
                                  const float* kv_scale, int64_t N_cap, const void* win_kv,
                                  int64_t L_raw, const int64_t* win_pos0, const float* sink,
                                  const void* q_rms_w, void* out, void* ws, size_t ws_bytes,
                                  void* stream);

/*
 * A paged classical KV cache ([P1''] 二、基础设施 (六): finished entries in blocks of a
 * multiple of lcm(m, m') raw tokens), as csa_state_append writes it: a pool of n_pages pages
 * of page_rows rows each; entry e of request b is row e % page_rows of page
 * page_table[b * max_pages + e / page_rows]. The logical capacity is
 * N_cap = page_rows * max_pages. Passed by pointer, read on the host during the call.
 */
typedef struct {
  csa_dtype fmt;              /* CSA_BF16 (pages [n_pages, page_rows, c]) or CSA_MIXED_FP8_BF16
                                 (pages [n_pages, page_rows, c + r] bytes)                  */
  const void* pages;          /* device                                                     */
  const void* scales;         /* CSA_MIXED_FP8_BF16 and CSA_FP8_E4M3_ROWSCALE: fp32
                                 [n_pages, page_rows]; CSA_MXFP4 keys: the e8m0 exponent
                                 blocks as csa_state_append writes them; else NULL          */
  const int32_t* page_table;  /* device int32 [B, max_pages]                               */
  int32_t n_pages, page_rows, max_pages;
} csa_paged_kv;

/*
 * Stage 4 over a paged cache: as csa_sparse_mqa / hca_dense_mqa with io = CSA_BF16 (the
 * mixed format as in csa_sparse_mqa_mixed_kv), reading each cache row through the page
 * table. An entry whose page id lies outside [0, n_pages) is skipped and leaves device
 * error code 205 for csa_device_error(). The window may be the state cache's ring
 * (csa_state_append's win_ring): pass win_pos0 = NULL and L_raw = n_win, one query per
 * request (T = 1); window position p is then read from row p mod n_win. Tensor-core attention only (c = 512, n_heads a
 * multiple of 64; mixed rows: rope_dims a multiple of 16 in (0, 512)), else
 * CSA_ERR_UNSUPPORTED. Workspace: csa_workspace_size() with N_cap = page_rows * max_pages.
 */
csa_status csa_sparse_mqa_paged(const csa_params* p, int32_t B, int32_t T, const void* q,
                                const int64_t* q_pos, const csa_paged_kv* kv, const int32_t* idx,
                                const void* win_kv, int64_t L_raw, const int64_t* win_pos0,
                                const float* sink, const void* q_rms_w, void* out, void* ws,
                                size_t ws_bytes, void* stream);
csa_status hca_dense_mqa_paged(const csa_params* p, int32_t B, int32_t T, const void* q,
                               const int64_t* q_pos, const csa_paged_kv* kv, const void* win_kv,
                               int64_t L_raw, const int64_t* win_pos0, const float* sink,
                               const void* q_rms_w, void* out, void* ws, size_t ws_bytes,
                               void* stream);

/*
 * Stages 2 + 3 over indexer keys kept in a page pool (the compressed indexer keys of the
 * state cache, [P1''] 二(六)): as csa_index_topk, the keys of request b read through the page
 * table; page_rows is a multiple of 128 and N_cap = page_rows * max_pages. keys->fmt:
 *   CSA_BF16: pages [n_pages, page_rows, 128] bf16; qI bf16 [B, T, 64, 128], qI_scale NULL;
 *   CSA_FP8_E4M3_ROWSCALE: e4m3 pages, scales fp32 [n_pages, page_rows]; qI as for bf16;
 *   CSA_MXFP4 ([P1'] 二(四)): pages [n_pages, page_rows, 64] e2m1 pairs and their e8m0
 *     exponent blocks, the layout csa_state_append writes with out_fmt = CSA_MXFP4 (a page is
 *     page_rows / 128 blocks, each laid out as for csa_index_scores); qI and qI_scale in
 *     MXFP4 as for csa_index_topk; at most 1024 queries per call.
 * bf16_scores = 1 selects on BF16 index scores as csa_index_topk_bf16 does. out_scores (fp32,
 * or bf16 with bf16_scores) may be NULL. A visible key whose page id lies outside the pool
 * reads pool row 0 and leaves device error code 309 (FP8 / bf16 keys) or 107 (MXFP4 keys).
 * Workspace: csa_workspace_size() with CSA_WS_INDEX_TOPK or CSA_WS_INDEX_TOPK_BF16.
 */
csa_status csa_index_topk_paged(const csa_params* p, int32_t B, int32_t T,
                                const csa_paged_kv* keys, const void* qI, const void* qI_scale,
                                const float* w, const int64_t* q_pos, int32_t bf16_scores,
                                int32_t* out_idx, void* out_scores, void* ws, size_t ws_bytes,
                                void* stream);

/*
 * The CSA layer over the state cache's paged caches: csa_index_topk_paged on `keys`
 * (optionally with BF16 index scores), then the sparse MQA over `kv` (bf16 or mixed rows,
 * as csa_sparse_mqa_paged), in one call with the decode chain of csa_forward. io = bf16 for
 * q [B, T, H, c], the window and out; qI (and qI_scale for MXFP4 keys) as for
 * csa_index_topk_paged with keys->fmt; w f32 [B, T, 64]. Both pools
 * cover N_cap = page_rows * max_pages entries. The window is a linear buffer with win_pos0,
 * or the state cache's ring (win_pos0 = NULL, L_raw = n_win, T = 1) as in
 * csa_sparse_mqa_paged. out_idx [B, T, k]; out_scores (fp32, or bf16 with bf16_scores) may
 * be NULL. Workspace: csa_workspace_size(..., CSA_WS_FORWARD, ...) with that N_cap.
 */
csa_status csa_forward_paged(const csa_params* p, int32_t B, int32_t T, const csa_paged_kv* kv,
                             const csa_paged_kv* keys, int32_t bf16_scores, const void* qI,
                             const void* qI_scale, const float* w, const void* q,
                             const void* q_rms_w,
                             const int64_t* q_pos, const void* win_kv, int64_t L_raw,
                             const int64_t* win_pos0, const float* sink, int32_t* out_idx,
                             void* out_scores, void* out, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * The hand-over from a prefill chunk to decode over the state cache ([P1''] 二(六)):
 *   csa_compress_paged: as csa_compress, writing entry first_entry + i of request b into row
 *     (first_entry + i) % page_rows of page page_table[b, (first_entry + i) / page_rows] of
 *     out_pages (fmt = io; N_cap = page_rows * max_pages). An entry whose page id lies
 *     outside the pool is skipped and leaves device error code 331.
 *   csa_state_resume: copies the chunk's last raw rows (Ca, Za, Cb, Zb [B, n_tok, c]; the
 *     chunk is tokens first_tok .. first_tok + n_tok - 1) into their slots of `state` and its
 *     last n_win window rows (win_rows [B, n_tok, c], final form; NULL with win_ring NULL)
 *     into `win_ring`, in the layouts of csa_state_append, so that appends continue at
 *     position first_tok + n_tok.
 */
csa_status csa_compress_paged(const csa_params* p, csa_dtype io, int32_t B, int64_t n_tok,
                              int64_t first_entry, const void* Ca, const void* Cb,
                              const void* Za, const void* Zb, const void* bias,
                              const void* prev_Cb, const void* prev_Zb, const void* kv_rms_w,
                              int32_t finalize, const csa_paged_kv* out_pages, void* stream);
csa_status csa_state_resume(const csa_params* p, csa_dtype io, int32_t B, int64_t first_tok,
                            int64_t n_tok, const void* Ca, const void* Cb, const void* Za,
                            const void* Zb, const void* win_rows, void* state, void* win_ring,
                            void* stream);

/*
 * Page allocation for the state cache's pools ([P1''] 二(六): finished entries in a
 * classical cache of blocks, each a multiple of lcm(m, m') raw tokens; [P4] §2: one logical
 * block of 128 raw tokens is 32 CSA entries or 1 HCA entry). One allocator serves one pool
 * of n_pages physical pages shared by B requests. It owns a host page table int32
 * [B, max_pages]: entry [b, k] is the physical page of request b's logical page k, or -1.
 * The caller copies the table (or the rows it changed) to the device before the launches
 * that read it. Free pages are handed out in order (first 0 .. n_pages-1, then pages given
 * back, in the order they were given back). Host memory only; not thread-safe.
 *
 *   csa_page_alloc_create: a pool with every page free and every table entry -1.
 *     *out = NULL on failure.
 *   csa_page_alloc_reserve: maps logical pages [0, n_logical) of request b, taking free
 *     pages for those not yet mapped (mapped ones stay). CSA_ERR_NO_PAGES, with nothing
 *     taken, when too few are free.
 *   csa_page_alloc_release: gives all of request b's pages back; its row becomes -1.
 *   csa_page_alloc_table: the host table [B, max_pages] (valid until destroy).
 *   csa_page_alloc_free_pages / csa_page_alloc_mapped: free pages in the pool / logical pages
 *     mapped for request b (-1 for an invalid handle or b).
 *   csa_state_pages_needed: logical pages that hold the entries of a request's first n_tok
 *     tokens, ceil(floor(n_tok / m) / page_rows); reserving that many before appending the
 *     token at position n_tok - 1 maps the page its entry goes to (-1 for invalid sizes).
 */
typedef struct csa_page_alloc csa_page_alloc;
csa_status csa_page_alloc_create(int32_t n_pages, int32_t B, int32_t max_pages,
                                 csa_page_alloc** out);
void csa_page_alloc_destroy(csa_page_alloc* a);
csa_status csa_page_alloc_reserve(csa_page_alloc* a, int32_t b, int32_t n_logical);
csa_status csa_page_alloc_release(csa_page_alloc* a, int32_t b);
const int32_t* csa_page_alloc_table(const csa_page_alloc* a);
int32_t csa_page_alloc_free_pages(const csa_page_alloc* a);
int32_t csa_page_alloc_mapped(const csa_page_alloc* a, int32_t b);
int32_t csa_state_pages_needed(int32_t m, int32_t page_rows, int64_t n_tok);

/*
 * Entries given as rows into a page pool in a storage format: the rows [B, n, c] (io =
 * CSA_F32 or CSA_BF16; e.g. a prefill chunk's entries from csa_compress) are entries
 * first_entry .. first_entry + n - 1 of every request, stored in out_pages->fmt exactly as
 * csa_state_append stores a finished row: the io dtype, CSA_FP8_E4M3_ROWSCALE (scales fp32
 * [n_pages, page_rows]), CSA_MXFP4 (c = 128, page_rows a multiple of 128; exponent blocks
 * as for csa_state_append) or CSA_MIXED_FP8_BF16 (0 < p->rope_dims < c). This is the
 * prefill -> decode hand-over for pools kept in a quantised format ([P1''] 二(六); [P1']
 * 二(四) for the FP4 indexer keys). An entry whose page id lies outside the pool is skipped
 * and leaves device error code 325 (324: its logical page is past the table, which the host
 * check rules out).
 */
csa_status csa_encode_paged(const csa_params* p, csa_dtype io, int32_t B, int64_t n,
                            int64_t first_entry, const void* rows,
                            const csa_paged_kv* out_pages, void* stream);

/* Inputs of the fused CSA layer call. Pointers as in the stage calls above. */
typedef struct {
  /* optional compression of a new chunk into kv_cache (skipped when Ca == NULL) */
  int64_t n_tok, first_entry;
  const void *Ca, *Cb, *Za, *Zb, *bias, *prev_Cb, *prev_Zb, *kv_rms_w;
  /* indexer */
  csa_dtype idx_dtype;
  const void *qI, *qI_scale;
  const float* w;
  const void *KI, *KI_scale;
  /* attention */
  const void* q;
  const void* q_rms_w;
  const int64_t* q_pos;
  void* kv_cache;
  int64_t N_cap;
  const void* win_kv;
  int64_t L_raw;
  const int64_t* win_pos0;
  const float* sink;
  /* outputs */
  int32_t* out_idx;  /* [B,T,k], required */
  float* out_scores; /* [B,T,N_cap] or NULL */
  void* out;         /* [B,T,H,c] */
} csa_forward_args;

/*
 * The CSA layer's hot path in one call: [compress the chunk into kv_cache] -> index scores
 * -> top-k -> sparse MQA, queued on `stream` in that order. io is the dtype of q, KV rows,
 * chunk inputs and out.
 */
csa_status csa_forward(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                       const csa_forward_args* a, void* ws, size_t ws_bytes, void* stream);

/*
 * Bytes of workspace the call `entry` needs for these sizes (0 if none). Returns 0 and
 * sets csa_last_error() on invalid sizes. kdt: the indexer key format (for the index calls).
 */
size_t csa_workspace_size(const csa_params* p, int32_t entry, csa_dtype kdt, int32_t B,
                          int32_t T, int64_t N_cap);

/*
 * Grouped output projection ([P1] 一(三)1(4) 分组输出投影; 2(2) for HCA) of Q queries: the
 * H = p->n_heads head outputs of query q, o[q] bf16 [H * c] (head after head,
 * the attention's out), are split into g groups of H/g heads; group i's c*H/g values times
 * w_grp[i] (bf16 [c*H/g, d_g]) give the intermediate o'[q, i*d_g .. (i+1)*d_g-1], and the
 * g*d_g intermediate values times w_out (bf16 [g*d_g, d]) give out[q] (bf16 [d]). Row
 * vectors multiply matrices from the left (x . W). Sums are fp32 over splits of the rows,
 * added in a fixed order (the intermediate stays fp32); the result is rounded to bf16 once.
 * Decode (Q < 128): each weight byte carries ~Q flops, so the call streams the weights from
 * HBM on CUDA cores, 16 queries per pass; sums stay fp32 until the final rounding.
 * Prefill (Q >= 128): two tcgen05 bf16 GEMMs with fp32 accumulation; the intermediate is
 * stored once in bf16 (needs c*H/g and g*d_g multiples of 64, d_g and d >= 64, else
 * CSA_ERR_UNSUPPORTED). Needs d_g and d multiples of 8, n_heads a multiple of g, and o,
 * w_grp, w_out, out and ws 16-byte aligned (16-byte weight loads, tensor-map copies and
 * stores), else CSA_ERR_INVALID_ARG (CSA_ERR_WORKSPACE for ws).
 * Workspace: csa_grouped_out_proj_workspace_size().
 */
csa_status csa_grouped_out_proj(const csa_params* p, int32_t Q, int32_t g, int32_t d_g,
                                int32_t d, const void* o, const void* w_grp, const void* w_out,
                                void* out, void* ws, size_t ws_bytes, void* stream);
size_t csa_grouped_out_proj_workspace_size(const csa_params* p, int32_t Q, int32_t g,
                                           int32_t d_g, int32_t d);

/* Static text of a status code. */
const char* csa_status_string(csa_status s);

/* One-line reason of the last non-OK status returned on the calling thread ("" if none). */
const char* csa_last_error(void);

/*
 * Timing hook for measurement. After a call with count > 0, every launch of the
 * indexer-score kernel records before[i] on the call's stream right before it and after[i]
 * right after it, i = 0, 1, 2, ... modulo count (cudaEvent_t handles owned by the caller).
 * count = 0 clears the hook. Not thread-safe; meant for benchmarks.
 */
void csa_set_index_timing_events(void* const* before, void* const* after, int32_t count);

/*
 * Error word of the tensor-core kernels: every wait inside them is bounded (about a second);
 * a wait that runs out stores a nonzero code (the first one wins) and the kernel returns
 * early instead of hanging. csa_state_append also leaves a code for a request it skipped.
 * Codes by kernel family: 101-107 MXFP4 indexer (107: a page id outside the pool), 201-205
 * attention (205: a page id outside the pool), 301-309 FP8 / bf16 indexer (309: a page id
 * outside the pool), 321-323 state append, 324-325 encoding into pages, 331 paged
 * compression, 401-405 prefill output projection. Writes the code to *code (0 = none) and clears it. Synchronises the device.
 * Returns CSA_ERR_CUDA if the copy fails.
 */
csa_status csa_device_error(int32_t* code);

/* Library version string. */
const char* csa_version(void);

/*
 * Number of kernels this library has launched in the process so far (every entry point,
 * every device). Diagnostic: the difference across a region counts its launches.
 */
uint64_t csa_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
