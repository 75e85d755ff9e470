// C ABI of libcsa (declared in include/csa.h): host-side validation, workspace layout and
// dispatch to the stage kernels. Nothing is launched unless every argument checks out.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "out_proj.cuh"
#include "state_append.cuh"

namespace csa {
std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace csa

namespace {

thread_local char g_err[256] = "";

csa_status fail(csa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

csa_status ok() {
  g_err[0] = '\0';
  return CSA_OK;
}

csa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return CSA_OK;
  return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, ...)                                  \
  do {                                                      \
    if (!(cond)) return fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)
#define REQUIRE_PTR(p) REQUIRE((p) != nullptr && aligned16(p), "%s must be a non-NULL 16-byte aligned device pointer", #p)
#define OPTIONAL_PTR(p) REQUIRE((p) == nullptr || aligned16(p), "%s must be 16-byte aligned", #p)

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

csa_status check_params(const csa_params* p) {
  REQUIRE(p != nullptr, "params is NULL");
  REQUIRE(p->m >= 1, "m must be >= 1 (got %d)", p->m);
  REQUIRE(p->c >= 64 && p->c % 64 == 0, "c must be a positive multiple of 64 (got %d)", p->c);
  REQUIRE(p->rope_dims >= 0 && p->rope_dims <= p->c && p->rope_dims % 2 == 0,
          "rope_dims must be even and in [0, c] (got %d)", p->rope_dims);
  REQUIRE(std::isfinite(p->rms_eps) && p->rms_eps >= 0.f, "rms_eps must be finite and >= 0");
  REQUIRE(std::isfinite(p->rope_base) && p->rope_base > 0.f, "rope_base must be > 0");
  REQUIRE(std::isfinite(p->sm_scale), "sm_scale must be finite");
  REQUIRE(p->n_win >= 0, "n_win must be >= 0");
  return CSA_OK;
}

csa_status check_attn(const csa_params* p) {
  REQUIRE(p->n_heads >= 1, "n_heads must be >= 1");
  REQUIRE(p->n_heads <= 16 || p->n_heads % 16 == 0,
          "n_heads must be <= 16 or a multiple of 16 (got %d)", p->n_heads);
  if (p->c > 512) return fail(CSA_ERR_UNSUPPORTED, "attention supports c <= 512 (got %d)", p->c);
  return CSA_OK;
}

csa_status check_index(const csa_params* p, csa_dtype kdt) {
  REQUIRE(p->n_idx_heads >= 1, "n_idx_heads must be >= 1");
  REQUIRE(p->d_idx >= 32 && p->d_idx % 32 == 0, "d_idx must be a positive multiple of 32");
  REQUIRE(kdt == CSA_F32 || kdt == CSA_BF16 || kdt == CSA_FP8_E4M3_ROWSCALE || kdt == CSA_MXFP4,
          "unknown indexer key dtype %d", (int)kdt);
  const size_t qbytes = (size_t)p->n_idx_heads * p->d_idx * 4 + p->n_idx_heads * 4;
  if (qbytes > 48 * 1024)
    return fail(CSA_ERR_UNSUPPORTED, "n_idx_heads * d_idx too large for the indexer (%d x %d)",
                p->n_idx_heads, p->d_idx);
  return CSA_OK;
}

csa_status check_topk(const csa_params* p) {
  REQUIRE(p->topk >= 1 && p->topk <= csa::kMaxTopk, "topk must be in [1, %d] (got %d)",
          csa::kMaxTopk, p->topk);
  return CSA_OK;
}

csa_status check_sizes(int32_t B, int32_t T, int64_t N_cap) {
  REQUIRE(B >= 0 && T >= 0, "B and T must be >= 0");
  REQUIRE(N_cap >= 0 && N_cap <= INT32_MAX, "N_cap must be in [0, 2^31)");
  REQUIRE((int64_t)B * T <= 65535 * 64, "B*T too large");
  return CSA_OK;
}

float eff_scale(const csa_params* p) {
  return p->sm_scale > 0.f ? p->sm_scale : 1.0f / std::sqrt((float)p->c);
}

#define TRY(x)                              \
  do {                                      \
    csa_status _s = (x);                    \
    if (_s != CSA_OK) return _s;            \
  } while (0)

struct TimingHook {
  std::vector<cudaEvent_t> before, after;
  size_t next = 0;
};
TimingHook g_timing;

csa::MqaArgs make_mqa(const csa_params* p, int32_t B, int32_t T, const void* q,
                      const int64_t* q_pos, const void* kv, int64_t N_cap, const int32_t* idx,
                      int k, const void* win, int64_t L_raw, const int64_t* pos0,
                      const float* sink, const void* q_rms_w, void* out) {
  csa::MqaArgs a{};
  a.B = B; a.T = T; a.m = p->m; a.H = p->n_heads; a.c = p->c; a.rope_dims = p->rope_dims;
  a.n_win = p->n_win; a.k = k; a.n_cap = N_cap; a.l_raw = L_raw; a.rope_base = p->rope_base;
  a.eps = p->rms_eps; a.scale = eff_scale(p); a.q = q; a.kv = kv; a.win = win;
  a.q_rms_w = q_rms_w; a.idx = idx; a.q_pos = q_pos; a.win_pos0 = pos0; a.sink = sink;
  a.out = out;
  return a;
}

csa_status check_mqa_args(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                          const void* q, const int64_t* q_pos, const void* kv, int64_t N_cap,
                          const void* win, int64_t L_raw, const int64_t* pos0,
                          const float* sink, const void* q_rms_w, const void* out,
                          bool ring_ok = false) {
  TRY(check_params(p));
  TRY(check_attn(p));
  TRY(check_sizes(B, T, N_cap));
  REQUIRE(io == CSA_F32 || io == CSA_BF16, "attention io dtype must be CSA_F32 or CSA_BF16");
  REQUIRE(L_raw >= 0, "L_raw must be >= 0");
  if ((int64_t)B * T == 0) return CSA_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(q_pos);
  REQUIRE_PTR(out);
  if (N_cap > 0) REQUIRE_PTR(kv);
  if (p->n_win > 0) {
    REQUIRE(L_raw >= 1, "n_win > 0 needs window rows (L_raw >= 1)");
    REQUIRE_PTR(win);
    if (ring_ok && pos0 == nullptr) {  // the state cache's window ring
      REQUIRE(L_raw == p->n_win, "a window ring holds n_win rows (L_raw = n_win)");
      REQUIRE(T == 1, "a window ring serves one query per request (T = 1)");
    } else {
      REQUIRE_PTR(pos0);
    }
  }
  OPTIONAL_PTR(sink);
  OPTIONAL_PTR(q_rms_w);
  return CSA_OK;
}

csa_status check_index_args(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                            int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                            const void* KI, const void* KI_scale, const int64_t* q_pos) {
  TRY(check_params(p));
  TRY(check_index(p, kdt));
  TRY(check_sizes(B, T, N_cap));
  if ((int64_t)B * T == 0) return CSA_OK;
  REQUIRE_PTR(qI);
  REQUIRE_PTR(w);
  REQUIRE_PTR(q_pos);
  if (N_cap > 0) REQUIRE_PTR(KI);
  if (kdt == CSA_FP8_E4M3_ROWSCALE && N_cap > 0) REQUIRE_PTR(KI_scale);
  if (kdt == CSA_MXFP4) {
    REQUIRE_PTR(qI_scale);
    if (N_cap > 0) REQUIRE_PTR(KI_scale);
    if (p->n_idx_heads != 64 || p->d_idx != 128)
      return fail(CSA_ERR_UNSUPPORTED, "MXFP4 keys need 64 indexer heads of dim 128");
    REQUIRE(N_cap % 128 == 0, "MXFP4 key caches hold whole 128-key scale blocks (N_cap %% 128)");
    REQUIRE((int64_t)B * T <= 1024, "MXFP4 indexer takes at most 1024 queries per call");
  }
  return CSA_OK;
}

// csa_forward with the tensor-core attention: the top-k kernel also prepares the
// attention's q_hat (bf16 [B*T][H][c]) in the workspace
bool forward_qhat(const csa_params* p, int32_t B, int32_t T, int64_t N_cap) {
  csa::MqaArgs m = make_mqa(p, B, T, nullptr, nullptr, nullptr, N_cap, nullptr, p->topk, nullptr,
                            0, nullptr, nullptr, nullptr, nullptr);
  return csa::mqa_tc_supported(m, true) && p->rope_dims <= 128;
}
size_t qhat_bytes(const csa_params* p, int32_t B, int32_t T, int64_t N_cap) {
  return forward_qhat(p, B, T, N_cap)
             ? round_up((size_t)B * T * (size_t)p->n_heads * (size_t)p->c * 2)
             : 0;
}

csa::IndexArgs make_index(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                          int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                          const void* KI, const void* KI_scale, const int64_t* q_pos,
                          float* scores) {
  csa::IndexArgs a{};
  a.B = B; a.T = T; a.m = p->m; a.n_idx_heads = p->n_idx_heads; a.d_idx = p->d_idx;
  a.kdt = (int)kdt; a.n_cap = N_cap; a.qI = qI; a.qI_scale = qI_scale; a.KI = KI;
  a.KI_scale = KI_scale; a.w = w; a.q_pos = q_pos; a.scores = scores;
  return a;
}

size_t scores_bytes(int32_t B, int32_t T, int64_t N_cap) {
  return round_up((size_t)B * T * (size_t)N_cap * sizeof(float));
}

// index scores, then top-k; for few long rows the indexer also fills the top-k histogram
csa_status index_then_topk(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                           int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                           const void* KI, const void* KI_scale, const int64_t* q_pos,
                           float* scores, const csa::TopkArgs& t, void* topk_ws,
                           size_t topk_bytes, cudaStream_t st, void* scores16 = nullptr,
                           const csa_paged_kv* key_pages = nullptr) {
  bool hist_done = false;
  const bool decode = csa::topk_decode_path(B, T, N_cap, p->topk);
  if (N_cap > 0) {
    auto ia = make_index(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, scores);
    ia.scores16 = scores16;
    if (key_pages != nullptr) {
      ia.page_table = key_pages->page_table;
      ia.page_rows = key_pages->page_rows;
      ia.max_pages = key_pages->max_pages;
      ia.n_pages = key_pages->n_pages;
    }
    if (decode) {
      const csa::TopkDecodeArgs da = csa::topk_decode_args(t, topk_ws);
      TRY(cuda_status(csa::topk_decode_clear(da, st), "top-k clear"));
      ia.hist = da.hist;
    }
    TRY(cuda_status(csa::launch_index_scores(ia, st, &hist_done), "index scores"));
  }
  TRY(cuda_status(csa::launch_topk(t, topk_ws, topk_bytes, st, hist_done), "top-k"));
  return CSA_OK;
}

}  // namespace

namespace csa {
void timing_before(cudaStream_t st) {
  if (!g_timing.before.empty())
    cudaEventRecord(g_timing.before[g_timing.next % g_timing.before.size()], st);
}
void timing_after(cudaStream_t st) {
  if (!g_timing.after.empty()) {
    cudaEventRecord(g_timing.after[g_timing.next % g_timing.after.size()], st);
    ++g_timing.next;
  }
}
}  // namespace csa

extern "C" {

const char* csa_version(void) { return "libcsa 0.1 (sm_100a)"; }

const char* csa_last_error(void) { return g_err; }

csa_status csa_device_error(int32_t* code) {
  REQUIRE(code != nullptr, "code is NULL");
  int words[6] = {0, 0, 0, 0, 0, 0};
  TRY(cuda_status(csa::index_mxf4_device_error(&words[0]), "device error word"));
  TRY(cuda_status(csa::mqa_tc_device_error(&words[1]), "device error word"));
  TRY(cuda_status(csa::index_bf16_device_error(&words[2]), "device error word"));
  TRY(cuda_status(csa::state_append_device_error(&words[3]), "device error word"));
  TRY(cuda_status(csa::out_proj_tc_device_error(&words[4]), "device error word"));
  TRY(cuda_status(csa::compress_device_error(&words[5]), "device error word"));
  *code = 0;
  for (int w : words)
    if (*code == 0) *code = w;
  return ok();
}

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_NO_PAGES: return "CSA_ERR_NO_PAGES";
  }
  return "CSA_ERR_UNKNOWN";
}

void csa_set_index_timing_events(void* const* before, void* const* after, int32_t count) {
  g_timing.before.clear();
  g_timing.after.clear();
  g_timing.next = 0;
  if (count <= 0 || before == nullptr || after == nullptr) return;
  for (int32_t i = 0; i < count; ++i) {
    g_timing.before.push_back(static_cast<cudaEvent_t>(before[i]));
    g_timing.after.push_back(static_cast<cudaEvent_t>(after[i]));
  }
}

size_t csa_workspace_size(const csa_params* p, int32_t entry, csa_dtype kdt, int32_t B,
                          int32_t T, int64_t N_cap) {
  if (check_params(p) != CSA_OK || check_sizes(B, T, N_cap) != CSA_OK) return 0;
  (void)kdt;
  const size_t topk_ws = round_up(csa::topk_workspace_bytes(B, T, N_cap, p->topk));
  csa::MqaArgs m = make_mqa(p, B, T, nullptr, nullptr, nullptr, N_cap, nullptr, p->topk,
                            nullptr, 0, nullptr, nullptr, nullptr, nullptr);
  switch (entry) {
    case CSA_WS_INDEX_TOPK:
      return scores_bytes(B, T, N_cap) + topk_ws;
    case CSA_WS_INDEX_TOPK_BF16:
      return round_up((size_t)B * T * (size_t)N_cap * 2) + topk_ws;
    case CSA_WS_TOPK:
      return topk_ws;
    case CSA_WS_SPARSE_MQA:
      return round_up(csa::mqa_workspace_bytes(m));
    case CSA_WS_HCA_MQA:
      m.k = 0;
      return round_up(csa::mqa_workspace_bytes(m));
    case CSA_WS_FORWARD:
      return scores_bytes(B, T, N_cap) + topk_ws + round_up(csa::mqa_workspace_bytes(m)) +
             qhat_bytes(p, B, T, N_cap);
    default:
      fail(CSA_ERR_INVALID_ARG, "unknown workspace entry %d", entry);
      return 0;
  }
}

namespace {
csa_status compress_impl(const csa_params* p, csa_dtype io, int32_t B, int64_t n_tok,
                         int64_t first_entry, int64_t n_cap, const void* Ca, const void* Cb,
                         const void* Za, const void* Zb, const void* bias, const void* prev_Cb,
                         const void* prev_Zb, const void* kv_rms_w, int32_t finalize,
                         void* out_cache, const csa_paged_kv* pages, void* stream) {
  TRY(check_params(p));
  REQUIRE(io == CSA_F32 || io == CSA_BF16, "compression io dtype must be CSA_F32 or CSA_BF16");
  REQUIRE(B >= 0 && B <= 65535, "B must be in [0, 65535]");
  REQUIRE(n_tok >= 0 && n_tok % p->m == 0, "n_tok must be a non-negative multiple of m");
  REQUIRE(first_entry >= 0 && n_cap >= 0 && first_entry + n_tok / p->m <= n_cap,
          "first_entry + n_tok/m must not exceed n_cap");
  REQUIRE(n_tok / p->m <= INT32_MAX, "too many entries");
  REQUIRE(p->overlap == 0 || p->overlap == 1, "overlap must be 0 or 1");
  REQUIRE(finalize == 0 || finalize == 1, "finalize must be 0 or 1");
  REQUIRE((prev_Cb == nullptr) == (prev_Zb == nullptr), "prev_Cb and prev_Zb go together");
  if (B == 0 || n_tok == 0) return ok();
  REQUIRE_PTR(Ca);
  REQUIRE_PTR(Za);
  REQUIRE_PTR(bias);
  REQUIRE_PTR(out_cache);
  if (p->overlap) {
    REQUIRE_PTR(Cb);
    REQUIRE_PTR(Zb);
    OPTIONAL_PTR(prev_Cb);
    OPTIONAL_PTR(prev_Zb);
  } else {
    REQUIRE(Cb == nullptr && Zb == nullptr && prev_Cb == nullptr,
            "HCA compression (overlap=0) takes no b-branch inputs");
  }
  OPTIONAL_PTR(kv_rms_w);
  csa::CompressArgs a{};
  a.B = B; a.m = p->m; a.c = p->c; a.overlap = p->overlap; a.rope_dims = p->rope_dims;
  a.finalize = finalize; a.n_tok = n_tok; a.first_entry = first_entry; a.n_cap = n_cap;
  a.rope_base = p->rope_base; a.eps = p->rms_eps; a.Ca = Ca; a.Cb = Cb; a.Za = Za; a.Zb = Zb;
  a.bias = bias; a.prev_Cb = prev_Cb; a.prev_Zb = prev_Zb; a.rms_w = kv_rms_w; a.out = out_cache;
  csa::CompressPages pg{};
  if (pages != nullptr)
    pg = csa::CompressPages{pages->page_table, pages->page_rows, pages->max_pages, pages->n_pages};
  TRY(cuda_status(csa::launch_compress(a, io == CSA_BF16, (cudaStream_t)stream,
                                       pages != nullptr ? &pg : nullptr),
                  "compress"));
  return ok();
}
}  // namespace

csa_status csa_compress(const csa_params* p, csa_dtype io, int32_t B, int64_t n_tok,
                        int64_t first_entry, int64_t n_cap, const void* Ca, const void* Cb,
                        const void* Za, const void* Zb, const void* bias, const void* prev_Cb,
                        const void* prev_Zb, const void* kv_rms_w, int32_t finalize,
                        void* out_cache, void* stream) {
  return compress_impl(p, io, B, n_tok, first_entry, n_cap, Ca, Cb, Za, Zb, bias, prev_Cb,
                       prev_Zb, kv_rms_w, finalize, out_cache, nullptr, stream);
}

csa_status csa_compress_paged(const csa_params* p, csa_dtype io, int32_t B, int64_t n_tok,
                              int64_t first_entry, const void* Ca, const void* Cb,
                              const void* Za, const void* Zb, const void* bias,
                              const void* prev_Cb, const void* prev_Zb, const void* kv_rms_w,
                              int32_t finalize, const csa_paged_kv* out_pages, void* stream) {
  REQUIRE(out_pages != nullptr, "page descriptor is NULL");
  REQUIRE(out_pages->fmt == io, "the pages hold rows in the io dtype");
  REQUIRE(out_pages->n_pages >= 1 && out_pages->page_rows >= 1 && out_pages->max_pages >= 1,
          "n_pages, page_rows and max_pages must be >= 1");
  REQUIRE_PTR(out_pages->page_table);
  const int64_t n_cap = (int64_t)out_pages->page_rows * out_pages->max_pages;
  return compress_impl(p, io, B, n_tok, first_entry, n_cap, Ca, Cb, Za, Zb, bias, prev_Cb,
                       prev_Zb, kv_rms_w, finalize, const_cast<void*>(out_pages->pages),
                       out_pages, stream);
}

csa_status csa_state_resume(const csa_params* p, csa_dtype io, int32_t B, int64_t first_tok,
                            int64_t n_tok, const void* Ca, const void* Cb, const void* Za,
                            const void* Zb, const void* win_rows, void* state, void* win_ring,
                            void* stream) {
  TRY(check_params(p));
  REQUIRE(io == CSA_F32 || io == CSA_BF16, "state io dtype must be CSA_F32 or CSA_BF16");
  REQUIRE(B >= 0 && B <= 65535, "B must be in [0, 65535]");
  REQUIRE(first_tok >= 0 && n_tok >= 0, "first_tok and n_tok must be >= 0");
  REQUIRE(p->overlap == 0 || p->overlap == 1, "overlap must be 0 or 1");
  REQUIRE((win_rows == nullptr) == (win_ring == nullptr), "win_rows and win_ring go together");
  REQUIRE(win_ring == nullptr || p->n_win >= 1, "a window ring needs n_win >= 1");
  if (p->overlap) {
    REQUIRE_PTR(Cb);
    REQUIRE_PTR(Zb);
  } else {
    REQUIRE(Cb == nullptr && Zb == nullptr, "HCA (overlap=0) takes no b-branch rows");
  }
  if (B == 0 || n_tok == 0) return ok();
  REQUIRE_PTR(Ca);
  REQUIRE_PTR(Za);
  REQUIRE_PTR(state);
  OPTIONAL_PTR(win_rows);
  OPTIONAL_PTR(win_ring);
  csa::state::Args a{};
  a.B = B; a.m = p->m; a.c = p->c; a.overlap = p->overlap; a.n_win = p->n_win;
  a.Ca = Ca; a.Cb = Cb; a.Za = Za; a.Zb = Zb; a.win_row = win_rows; a.state = state;
  a.win_ring = win_ring;
  TRY(cuda_status(csa::launch_state_resume(a, io == CSA_BF16, first_tok, n_tok,
                                           (cudaStream_t)stream), "state resume"));
  return ok();
}

csa_status csa_state_append(const csa_params* p, csa_dtype io, int32_t B, const int64_t* pos,
                            const void* Ca, const void* Cb, const void* Za, const void* Zb,
                            const void* win_row, const void* bias, const void* kv_rms_w,
                            int32_t finalize, void* state, void* win_ring, csa_dtype out_fmt,
                            void* pages, void* page_scales, int32_t n_pages, int32_t page_rows,
                            const int32_t* page_table, int32_t max_pages, void* stream) {
  TRY(check_params(p));
  REQUIRE(io == CSA_F32 || io == CSA_BF16, "state io dtype must be CSA_F32 or CSA_BF16");
  REQUIRE(p->c <= 4096, "state append supports c <= 4096 (got %d)", p->c);
  REQUIRE(out_fmt == io || out_fmt == CSA_FP8_E4M3_ROWSCALE || out_fmt == CSA_MXFP4 ||
              out_fmt == CSA_MIXED_FP8_BF16,
          "out_fmt must be the io dtype, CSA_FP8_E4M3_ROWSCALE, CSA_MXFP4 or CSA_MIXED_FP8_BF16");
  if (out_fmt == CSA_MIXED_FP8_BF16)
    REQUIRE(p->rope_dims > 0 && p->rope_dims < p->c && p->rope_dims % 16 == 0,
            "mixed rows need 0 < rope_dims < c and rope_dims a multiple of 16 (16-byte "
            "aligned rows, as the attention over mixed rows reads them)");
  if (out_fmt == CSA_MXFP4) {
    REQUIRE(p->c == 128, "MXFP4 rows are indexer keys of 128 values (c = %d)", p->c);
    REQUIRE(page_rows % 128 == 0, "MXFP4 pages hold whole 128-row exponent blocks");
  }
  REQUIRE(B >= 0 && B <= 65535, "B must be in [0, 65535]");
  REQUIRE(p->overlap == 0 || p->overlap == 1, "overlap must be 0 or 1");
  REQUIRE(finalize == 0 || finalize == 1, "finalize must be 0 or 1");
  REQUIRE(p->rope_dims / 2 <= 256, "rope_dims must be <= 512");
  REQUIRE(n_pages >= 1 && page_rows >= 1 && max_pages >= 1,
          "n_pages, page_rows and max_pages must be >= 1");
  REQUIRE((win_row == nullptr) == (win_ring == nullptr), "win_row and win_ring go together");
  REQUIRE(win_ring == nullptr || p->n_win >= 1, "a window ring needs n_win >= 1");
  if (p->overlap) {
    REQUIRE_PTR(Cb);
    REQUIRE_PTR(Zb);
  } else {
    REQUIRE(Cb == nullptr && Zb == nullptr, "HCA (overlap=0) takes no b-branch rows");
  }
  if (B == 0) return ok();
  REQUIRE_PTR(pos);
  REQUIRE_PTR(Ca);
  REQUIRE_PTR(Za);
  REQUIRE_PTR(bias);
  REQUIRE_PTR(state);
  REQUIRE_PTR(pages);
  REQUIRE_PTR(page_table);
  if (out_fmt != io) REQUIRE_PTR(page_scales);
  OPTIONAL_PTR(win_row);
  OPTIONAL_PTR(win_ring);
  OPTIONAL_PTR(kv_rms_w);
  csa::state::Args a{};
  a.B = B; a.m = p->m; a.c = p->c; a.overlap = p->overlap; a.rope_dims = p->rope_dims;
  a.finalize = finalize; a.n_win = p->n_win; a.n_pages = n_pages; a.page_rows = page_rows;
  a.max_pages = max_pages; a.eps = p->rms_eps; a.pos = pos; a.Ca = Ca; a.Cb = Cb; a.Za = Za;
  a.Zb = Zb; a.win_row = win_row; a.bias = bias; a.rms_w = kv_rms_w; a.state = state;
  a.win_ring = win_ring; a.pages = pages; a.page_scales = page_scales;
  a.page_table = page_table;
  a.out = out_fmt == io                   ? csa::state::kOutIo
          : out_fmt == CSA_MXFP4          ? csa::state::kOutMxfp4
          : out_fmt == CSA_MIXED_FP8_BF16 ? csa::state::kOutMixed
                                          : csa::state::kOutFp8;
  for (int i = 0; i < p->rope_dims / 2; ++i)
    a.inv_freq[i] = csa::rope_inv_freq(i, p->rope_dims, (double)p->rope_base);
  TRY(cuda_status(csa::launch_state_append(a, io == CSA_BF16, (cudaStream_t)stream),
                  "state append"));
  return ok();
}

csa_status csa_encode_paged(const csa_params* p, csa_dtype io, int32_t B, int64_t n,
                            int64_t first_entry, const void* rows,
                            const csa_paged_kv* out_pages, void* stream) {
  TRY(check_params(p));
  REQUIRE(io == CSA_F32 || io == CSA_BF16, "rows must be CSA_F32 or CSA_BF16");
  REQUIRE(p->c <= 4096, "encoding supports c <= 4096 (got %d)", p->c);
  REQUIRE(out_pages != nullptr, "page descriptor is NULL");
  const csa_dtype fmt = out_pages->fmt;
  REQUIRE(fmt == io || fmt == CSA_FP8_E4M3_ROWSCALE || fmt == CSA_MXFP4 ||
              fmt == CSA_MIXED_FP8_BF16,
          "page format must be the io dtype, CSA_FP8_E4M3_ROWSCALE, CSA_MXFP4 or "
          "CSA_MIXED_FP8_BF16");
  if (fmt == CSA_MIXED_FP8_BF16)
    REQUIRE(p->rope_dims > 0 && p->rope_dims < p->c && p->rope_dims % 16 == 0,
            "mixed rows need 0 < rope_dims < c and rope_dims a multiple of 16 (16-byte "
            "aligned rows, as the attention over mixed rows reads them)");
  if (fmt == CSA_MXFP4) {
    REQUIRE(p->c == 128, "MXFP4 rows are indexer keys of 128 values (c = %d)", p->c);
    REQUIRE(out_pages->page_rows % 128 == 0, "MXFP4 pages hold whole 128-row exponent blocks");
  }
  REQUIRE(B >= 0 && B <= 65535, "B must be in [0, 65535]");
  REQUIRE(n >= 0 && n <= INT32_MAX && first_entry >= 0, "n and first_entry must be >= 0");
  REQUIRE(out_pages->n_pages >= 1 && out_pages->page_rows >= 1 && out_pages->max_pages >= 1,
          "n_pages, page_rows and max_pages must be >= 1");
  REQUIRE(first_entry + n <= (int64_t)out_pages->page_rows * out_pages->max_pages,
          "entries %lld .. %lld lie past the page table (%d pages of %d rows)",
          (long long)first_entry, (long long)(first_entry + n - 1), out_pages->max_pages,
          out_pages->page_rows);
  if ((int64_t)B * n == 0) return ok();
  REQUIRE_PTR(rows);
  REQUIRE_PTR(out_pages->pages);
  REQUIRE_PTR(out_pages->page_table);
  if (fmt != io) REQUIRE_PTR(out_pages->scales);
  csa::state::Args a{};
  a.B = B; a.m = p->m; a.c = p->c; a.overlap = p->overlap; a.rope_dims = p->rope_dims;
  a.n_pages = out_pages->n_pages; a.page_rows = out_pages->page_rows;
  a.max_pages = out_pages->max_pages; a.eps = p->rms_eps;
  a.pages = const_cast<void*>(out_pages->pages);
  a.page_scales = const_cast<void*>(out_pages->scales);
  a.page_table = out_pages->page_table;
  a.out = fmt == io                   ? csa::state::kOutIo
          : fmt == CSA_MXFP4          ? csa::state::kOutMxfp4
          : fmt == CSA_MIXED_FP8_BF16 ? csa::state::kOutMixed
                                      : csa::state::kOutFp8;
  TRY(cuda_status(csa::launch_encode_paged(a, io == CSA_BF16, rows, n, first_entry,
                                           (cudaStream_t)stream), "encode into pages"));
  return ok();
}

namespace {
csa_status check_out_proj(const csa_params* p, int32_t Q, int32_t g, int32_t d_g, int32_t d) {
  TRY(check_params(p));
  REQUIRE(Q >= 0, "Q must be >= 0");
  REQUIRE(p->n_heads >= 1 && g >= 1 && p->n_heads % g == 0,
          "n_heads (%d) must be a positive multiple of g (%d)", p->n_heads, g);
  REQUIRE(d_g >= 8 && d_g % 8 == 0 && d >= 8 && d % 8 == 0,
          "d_g and d must be positive multiples of 8 (got %d, %d)", d_g, d);
  REQUIRE((int64_t)p->c * p->n_heads <= (1 << 24) && (int64_t)g * d_g <= (1 << 24) &&
              d <= (1 << 24), "sizes too large");
  if (Q >= 128) {
    const csa::proj::Geom G = csa::out_proj_geom(Q, p->n_heads, p->c, g, d_g, d);
    if (!csa::out_proj_tc_shape_ok(G))
      return fail(CSA_ERR_UNSUPPORTED,
                  "grouped output projection of %d queries: the tensor-core form needs c*H/g "
                  "and g*d_g multiples of 64 and d_g, d >= 64", Q);
  }
  return CSA_OK;
}

// Queries per pass of the weight-streaming (decode) kernels, and the form a call takes.
constexpr int32_t kStreamQueries = 16;
bool out_proj_uses_tc(int32_t Q) { return Q >= 128; }
}  // namespace

size_t csa_grouped_out_proj_workspace_size(const csa_params* p, int32_t Q, int32_t g,
                                           int32_t d_g, int32_t d) {
  if (check_out_proj(p, Q, g, d_g, d) != CSA_OK || Q == 0) return 0;
  if (out_proj_uses_tc(Q))
    return csa::out_proj_tc_workspace_bytes(csa::out_proj_geom(Q, p->n_heads, p->c, g, d_g, d));
  const int32_t q = Q < kStreamQueries ? Q : kStreamQueries;
  return csa::out_proj_workspace_bytes(csa::out_proj_geom(q, p->n_heads, p->c, g, d_g, d));
}

csa_status csa_grouped_out_proj(const csa_params* p, int32_t Q, int32_t g, int32_t d_g,
                                int32_t d, const void* o, const void* w_grp, const void* w_out,
                                void* out, void* ws, size_t ws_bytes, void* stream) {
  TRY(check_out_proj(p, Q, g, d_g, d));
  if (Q == 0) return ok();
  REQUIRE_PTR(o);
  REQUIRE_PTR(w_grp);
  REQUIRE_PTR(w_out);
  REQUIRE_PTR(out);
  const size_t need = csa_grouped_out_proj_workspace_size(p, Q, g, d_g, d);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws))
    return fail(CSA_ERR_WORKSPACE, "grouped output projection needs %zu workspace bytes", need);
  csa::OutProjArgs a{};
  a.w_grp = static_cast<const __nv_bfloat16*>(w_grp);
  a.w_out = static_cast<const __nv_bfloat16*>(w_out);
  cudaStream_t st = (cudaStream_t)stream;
  if (out_proj_uses_tc(Q)) {  // prefill: two tensor-core GEMMs
    a.G = csa::out_proj_geom(Q, p->n_heads, p->c, g, d_g, d);
    a.o = static_cast<const __nv_bfloat16*>(o);
    a.out = static_cast<__nv_bfloat16*>(out);
    TRY(cuda_status(csa::launch_out_proj_tc(a, ws, st), "grouped output projection"));
    return ok();
  }
  // decode: weight streaming, at most kStreamQueries queries per pass
  for (int32_t q0 = 0; q0 < Q; q0 += kStreamQueries) {
    const int32_t q = Q - q0 < kStreamQueries ? Q - q0 : kStreamQueries;
    a.G = csa::out_proj_geom(q, p->n_heads, p->c, g, d_g, d);
    a.o = static_cast<const __nv_bfloat16*>(o) + (size_t)q0 * p->n_heads * p->c;
    a.out = static_cast<__nv_bfloat16*>(out) + (size_t)q0 * d;
    TRY(cuda_status(csa::launch_out_proj(a, ws, st), "grouped output projection"));
  }
  return ok();
}

csa_status csa_index_scores(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                            int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                            const void* KI, const void* KI_scale, const int64_t* q_pos,
                            float* out_scores, void* stream) {
  TRY(check_index_args(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos));
  if ((int64_t)B * T == 0 || N_cap == 0) return ok();
  REQUIRE_PTR(out_scores);
  auto a = make_index(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, out_scores);
  TRY(cuda_status(csa::launch_index_scores(a, (cudaStream_t)stream), "index scores"));
  return ok();
}

csa_status csa_topk(const csa_params* p, int32_t B, int32_t T, int64_t N_cap,
                    const float* scores, const int64_t* q_pos, int32_t* out_idx, void* ws,
                    size_t ws_bytes, void* stream) {
  TRY(check_params(p));
  TRY(check_topk(p));
  TRY(check_sizes(B, T, N_cap));
  if ((int64_t)B * T == 0) return ok();
  if (N_cap > 0) REQUIRE_PTR(scores);
  REQUIRE_PTR(q_pos);
  REQUIRE_PTR(out_idx);
  const size_t need = csa::topk_workspace_bytes(B, T, N_cap, p->topk);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(CSA_ERR_WORKSPACE, "top-k needs %zu workspace bytes", need);
  csa::TopkArgs a{};
  a.B = B; a.T = T; a.m = p->m; a.k = p->topk; a.n_cap = N_cap; a.scores = scores;
  a.q_pos = q_pos; a.out_idx = out_idx;
  TRY(cuda_status(csa::launch_topk(a, ws, ws_bytes, (cudaStream_t)stream), "top-k"));
  return ok();
}

csa_status csa_index_topk(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                          int64_t N_cap, const void* qI, const void* qI_scale, const float* w,
                          const void* KI, const void* KI_scale, const int64_t* q_pos,
                          int32_t* out_idx, float* out_scores, void* ws, size_t ws_bytes,
                          void* stream) {
  TRY(check_index_args(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos));
  TRY(check_topk(p));
  if ((int64_t)B * T == 0) return ok();
  REQUIRE_PTR(out_idx);
  OPTIONAL_PTR(out_scores);
  const size_t need = csa_workspace_size(p, CSA_WS_INDEX_TOPK, kdt, B, T, N_cap);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws))
    return fail(CSA_ERR_WORKSPACE, "index+top-k needs %zu workspace bytes (got %zu)", need,
                ws_bytes);
  char* base = static_cast<char*>(ws);
  float* scores = out_scores ? out_scores : reinterpret_cast<float*>(base);
  char* topk_ws = base + scores_bytes(B, T, N_cap);
  const size_t topk_bytes = need - scores_bytes(B, T, N_cap);
  cudaStream_t st = (cudaStream_t)stream;
  csa::TopkArgs t{};
  t.B = B; t.T = T; t.m = p->m; t.k = p->topk; t.n_cap = N_cap; t.scores = scores;
  t.q_pos = q_pos; t.out_idx = out_idx;
  TRY(index_then_topk(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, scores, t,
                      topk_ws, topk_bytes, st));
  return ok();
}

csa_status csa_index_topk_bf16(const csa_params* p, csa_dtype kdt, int32_t B, int32_t T,
                               int64_t N_cap, const void* qI, const void* qI_scale,
                               const float* w, const void* KI, const void* KI_scale,
                               const int64_t* q_pos, int32_t* out_idx, void* out_scores16,
                               void* ws, size_t ws_bytes, void* stream) {
  TRY(check_index_args(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos));
  TRY(check_topk(p));
  if ((int64_t)B * T == 0) return ok();
  REQUIRE_PTR(out_idx);
  OPTIONAL_PTR(out_scores16);
  {
    auto ia = make_index(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, nullptr);
    if (N_cap > 0 && !csa::index_bf16_tc_supported(ia) && !csa::index_mxf4_tc_supported(ia))
      return fail(CSA_ERR_UNSUPPORTED,
                  "BF16 index scores come from the tensor-core indexers (MXFP4, FP8 or bf16 "
                  "keys; 64 heads of 128, N_cap a multiple of 128)");
  }
  const size_t need = csa_workspace_size(p, CSA_WS_INDEX_TOPK_BF16, kdt, B, T, N_cap);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws))
    return fail(CSA_ERR_WORKSPACE, "index+top-k (bf16 scores) needs %zu workspace bytes", need);
  char* base = static_cast<char*>(ws);
  const size_t sb = round_up((size_t)B * T * (size_t)N_cap * 2);
  void* s16 = out_scores16 ? out_scores16 : base;
  csa::TopkArgs t{};
  t.B = B; t.T = T; t.m = p->m; t.k = p->topk; t.n_cap = N_cap; t.scores = nullptr;
  t.scores16 = s16; t.q_pos = q_pos; t.out_idx = out_idx;
  TRY(index_then_topk(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, nullptr, t,
                      base + sb, need - sb, (cudaStream_t)stream, s16));
  return ok();
}

namespace {

// the paged indexer-key descriptor: its format and pool sizes
csa_status check_paged_keys(const csa_paged_kv* keys) {
  REQUIRE(keys != nullptr, "paged key descriptor is NULL");
  REQUIRE(keys->fmt == CSA_BF16 || keys->fmt == CSA_FP8_E4M3_ROWSCALE || keys->fmt == CSA_MXFP4,
          "paged indexer keys must be CSA_BF16, CSA_FP8_E4M3_ROWSCALE or CSA_MXFP4");
  REQUIRE(keys->n_pages >= 1 && keys->max_pages >= 1 && keys->page_rows >= 1,
          "n_pages, page_rows and max_pages must be >= 1");
  REQUIRE((int64_t)keys->page_rows * keys->max_pages <= INT32_MAX,
          "page_rows * max_pages too large");
  REQUIRE_PTR(keys->page_table);
  return CSA_OK;
}

// the tensor-core indexer that reads paged keys of this format, or CSA_ERR_UNSUPPORTED
csa_status check_paged_index(const csa_params* p, const csa_paged_kv* keys, int32_t B,
                             int32_t T, const void* qI, const void* qI_scale, const float* w,
                             const int64_t* q_pos) {
  const int64_t N_cap = (int64_t)keys->page_rows * keys->max_pages;
  auto ia = make_index(p, keys->fmt, B, T, N_cap, qI, qI_scale, w, keys->pages, keys->scales,
                       q_pos, nullptr);
  ia.page_table = keys->page_table;
  ia.page_rows = keys->page_rows;
  ia.max_pages = keys->max_pages;
  ia.n_pages = keys->n_pages;
  if (!csa::index_bf16_tc_supported(ia) && !csa::index_mxf4_tc_supported(ia))
    return fail(CSA_ERR_UNSUPPORTED,
                "paged keys are read by the tensor-core indexers (64 heads of 128, page_rows a "
                "multiple of 128)");
  return CSA_OK;
}

}  // namespace

csa_status csa_index_topk_paged(const csa_params* p, int32_t B, int32_t T,
                                const csa_paged_kv* keys, const void* qI, const void* qI_scale,
                                const float* w, const int64_t* q_pos, int32_t bf16_scores,
                                int32_t* out_idx, void* out_scores, void* ws, size_t ws_bytes,
                                void* stream) {
  TRY(check_params(p));
  TRY(check_topk(p));
  TRY(check_paged_keys(keys));
  REQUIRE(bf16_scores == 0 || bf16_scores == 1, "bf16_scores must be 0 or 1");
  const int64_t N_cap = (int64_t)keys->page_rows * keys->max_pages;
  const csa_dtype kdt = keys->fmt;
  if (kdt != CSA_MXFP4) REQUIRE(qI_scale == nullptr, "qI_scale is for MXFP4 queries only");
  TRY(check_index_args(p, kdt, B, T, N_cap, qI, qI_scale, w, keys->pages, keys->scales, q_pos));
  if ((int64_t)B * T == 0) return ok();
  REQUIRE_PTR(out_idx);
  OPTIONAL_PTR(out_scores);
  TRY(check_paged_index(p, keys, B, T, qI, qI_scale, w, q_pos));
  const int entry = bf16_scores ? CSA_WS_INDEX_TOPK_BF16 : CSA_WS_INDEX_TOPK;
  const size_t need = csa_workspace_size(p, entry, kdt, B, T, N_cap);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws))
    return fail(CSA_ERR_WORKSPACE, "index+top-k (paged keys) needs %zu workspace bytes", need);
  char* base = static_cast<char*>(ws);
  const size_t sb = bf16_scores ? round_up((size_t)B * T * (size_t)N_cap * 2)
                                : scores_bytes(B, T, N_cap);
  void* sc = out_scores ? out_scores : base;
  csa::TopkArgs t{};
  t.B = B; t.T = T; t.m = p->m; t.k = p->topk; t.n_cap = N_cap; t.q_pos = q_pos;
  t.out_idx = out_idx;
  if (bf16_scores) t.scores16 = sc;
  else t.scores = static_cast<float*>(sc);
  TRY(index_then_topk(p, kdt, B, T, N_cap, qI, qI_scale, w, keys->pages, keys->scales, q_pos,
                      bf16_scores ? nullptr : static_cast<float*>(sc), t, base + sb, need - sb,
                      (cudaStream_t)stream, bf16_scores ? sc : nullptr, keys));
  return ok();
}

csa_status csa_sparse_mqa(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                          const void* q, const int64_t* q_pos, const void* kv_cache,
                          int64_t N_cap, const int32_t* idx, const void* win_kv, int64_t L_raw,
                          const int64_t* win_pos0, const float* sink, const void* q_rms_w,
                          void* out, void* ws, size_t ws_bytes, void* stream) {
  TRY(check_mqa_args(p, io, B, T, q, q_pos, kv_cache, N_cap, win_kv, L_raw, win_pos0, sink,
                     q_rms_w, out));
  TRY(check_topk(p));
  if ((int64_t)B * T == 0) return ok();
  REQUIRE_PTR(idx);
  auto a = make_mqa(p, B, T, q, q_pos, kv_cache, N_cap, idx, p->topk, win_kv, L_raw, win_pos0,
                    sink, q_rms_w, out);
  const size_t need = csa::mqa_workspace_bytes(a);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(CSA_ERR_WORKSPACE, "sparse MQA needs %zu workspace bytes", need);
  TRY(cuda_status(csa::launch_mqa(a, io == CSA_BF16, ws, ws_bytes, (cudaStream_t)stream),
                  "sparse MQA"));
  return ok();
}

csa_status hca_dense_mqa(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                         const void* q, const int64_t* q_pos, const void* kv_cache,
                         int64_t N_cap, const void* win_kv, int64_t L_raw,
                         const int64_t* win_pos0, const float* sink, const void* q_rms_w,
                         void* out, void* ws, size_t ws_bytes, void* stream) {
  TRY(check_mqa_args(p, io, B, T, q, q_pos, kv_cache, N_cap, win_kv, L_raw, win_pos0, sink,
                     q_rms_w, out));
  if ((int64_t)B * T == 0) return ok();
  auto a = make_mqa(p, B, T, q, q_pos, kv_cache, N_cap, nullptr, 0, win_kv, L_raw, win_pos0,
                    sink, q_rms_w, out);
  const size_t need = csa::mqa_workspace_bytes(a);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(CSA_ERR_WORKSPACE, "dense MQA needs %zu workspace bytes", need);
  TRY(cuda_status(csa::launch_mqa(a, io == CSA_BF16, ws, ws_bytes, (cudaStream_t)stream),
                  "dense MQA"));
  return ok();
}

namespace {
// Tensor-core attention over mixed-precision and / or paged cache rows.
struct KvLayout {
  bool mixed;
  const void* rows;            // contiguous cache [B, N_cap, ...] or page pool
  const float* scales;         // mixed: per-row scales (same indexing as rows)
  const int32_t* page_table;   // paged: [B, max_pages]; NULL: contiguous
  int32_t n_pages, page_rows, max_pages;
};

csa_status tc_mqa_ext(const char* what, const csa_params* p, int32_t B, int32_t T,
                      const void* q, const int64_t* q_pos, const KvLayout& kv, int64_t N_cap,
                      const int32_t* idx, int k, const void* win_kv, int64_t L_raw,
                      const int64_t* win_pos0, const float* sink, const void* q_rms_w,
                      void* out, void* ws, size_t ws_bytes, void* stream) {
  TRY(check_mqa_args(p, CSA_BF16, B, T, q, q_pos, kv.rows, N_cap, win_kv, L_raw, win_pos0, sink,
                     q_rms_w, out, kv.page_table != nullptr));
  if ((int64_t)B * T == 0) return ok();
  if (k > 0) REQUIRE_PTR(idx);
  if (kv.mixed && N_cap > 0) REQUIRE_PTR(kv.scales);
  if (kv.page_table != nullptr) REQUIRE_PTR(kv.page_table);
  auto a = make_mqa(p, B, T, q, q_pos, kv.rows, N_cap, idx, k, win_kv, L_raw, win_pos0, sink,
                    q_rms_w, out);
  const bool rope_ok = !kv.mixed ||
                       (p->rope_dims > 0 && p->rope_dims < p->c && p->rope_dims % 16 == 0);
  if (!rope_ok || !csa::mqa_tc_supported(a, true))
    return fail(CSA_ERR_UNSUPPORTED,
                "%s: needs the tensor-core attention (c = 512, n_heads a multiple of 64; "
                "mixed rows: rope_dims a multiple of 16 in (0, 512))", what);
  if (N_cap > 0) {  // no cache rows: nothing to widen or look up
    a.kv_scale = kv.mixed ? kv.scales : nullptr;
    a.page_table = kv.page_table;
    a.n_pages = kv.n_pages;
    a.page_rows = kv.page_rows;
    a.max_pages = kv.max_pages;
  }
  const size_t need = csa::mqa_workspace_bytes(a);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(CSA_ERR_WORKSPACE, "%s needs %zu workspace bytes", what, need);
  TRY(cuda_status(csa::launch_mqa(a, true, ws, ws_bytes, (cudaStream_t)stream), what));
  return ok();
}

csa_status paged_layout(const csa_paged_kv* kv, KvLayout* out, int64_t* N_cap) {
  REQUIRE(kv != nullptr, "paged KV descriptor is NULL");
  REQUIRE(kv->fmt == CSA_BF16 || kv->fmt == CSA_MIXED_FP8_BF16,
          "paged KV format must be CSA_BF16 or CSA_MIXED_FP8_BF16");
  REQUIRE(kv->n_pages >= 1 && kv->page_rows >= 1 && kv->max_pages >= 1,
          "n_pages, page_rows and max_pages must be >= 1");
  REQUIRE((int64_t)kv->page_rows * kv->max_pages <= INT32_MAX, "page_rows * max_pages too large");
  REQUIRE_PTR(kv->pages);
  REQUIRE_PTR(kv->page_table);
  if (kv->fmt == CSA_MIXED_FP8_BF16) REQUIRE_PTR(kv->scales);
  *out = KvLayout{kv->fmt == CSA_MIXED_FP8_BF16, kv->pages,
                  static_cast<const float*>(kv->scales), kv->page_table, kv->n_pages,
                  kv->page_rows, kv->max_pages};
  *N_cap = (int64_t)kv->page_rows * kv->max_pages;
  return CSA_OK;
}
}  // namespace

csa_status csa_sparse_mqa_mixed_kv(const csa_params* p, int32_t B, int32_t T, const void* q,
                                   const int64_t* q_pos, const void* kv_rows,
                                   const float* kv_scale, int64_t N_cap, const int32_t* idx,
                                   const void* win_kv, int64_t L_raw, const int64_t* win_pos0,
                                   const float* sink, const void* q_rms_w, void* out, void* ws,
                                   size_t ws_bytes, void* stream) {
  TRY(check_params(p));
  TRY(check_topk(p));
  const KvLayout kv{true, kv_rows, kv_scale, nullptr, 0, 0, 0};
  return tc_mqa_ext("sparse MQA (mixed KV)", p, B, T, q, q_pos, kv, N_cap, idx, p->topk, win_kv,
                    L_raw, win_pos0, sink, q_rms_w, out, ws, ws_bytes, stream);
}

csa_status hca_dense_mqa_mixed_kv(const csa_params* p, int32_t B, int32_t T, const void* q,
                                  const int64_t* q_pos, const void* kv_rows,
                                  const float* kv_scale, int64_t N_cap, const void* win_kv,
                                  int64_t L_raw, const int64_t* win_pos0, const float* sink,
                                  const void* q_rms_w, void* out, void* ws, size_t ws_bytes,
                                  void* stream) {
  TRY(check_params(p));
  const KvLayout kv{true, kv_rows, kv_scale, nullptr, 0, 0, 0};
  return tc_mqa_ext("dense MQA (mixed KV)", p, B, T, q, q_pos, kv, N_cap, nullptr, 0, win_kv,
                    L_raw, win_pos0, sink, q_rms_w, out, ws, ws_bytes, stream);
}

csa_status csa_sparse_mqa_paged(const csa_params* p, int32_t B, int32_t T, const void* q,
                                const int64_t* q_pos, const csa_paged_kv* kv, const int32_t* idx,
                                const void* win_kv, int64_t L_raw, const int64_t* win_pos0,
                                const float* sink, const void* q_rms_w, void* out, void* ws,
                                size_t ws_bytes, void* stream) {
  TRY(check_params(p));
  TRY(check_topk(p));
  KvLayout lay;
  int64_t N_cap = 0;
  TRY(paged_layout(kv, &lay, &N_cap));
  return tc_mqa_ext("sparse MQA (paged KV)", p, B, T, q, q_pos, lay, N_cap, idx, p->topk, win_kv,
                    L_raw, win_pos0, sink, q_rms_w, out, ws, ws_bytes, stream);
}

csa_status hca_dense_mqa_paged(const csa_params* p, int32_t B, int32_t T, const void* q,
                               const int64_t* q_pos, const csa_paged_kv* kv, const void* win_kv,
                               int64_t L_raw, const int64_t* win_pos0, const float* sink,
                               const void* q_rms_w, void* out, void* ws, size_t ws_bytes,
                               void* stream) {
  TRY(check_params(p));
  KvLayout lay;
  int64_t N_cap = 0;
  TRY(paged_layout(kv, &lay, &N_cap));
  return tc_mqa_ext("dense MQA (paged KV)", p, B, T, q, q_pos, lay, N_cap, nullptr, 0, win_kv,
                    L_raw, win_pos0, sink, q_rms_w, out, ws, ws_bytes, stream);
}

csa_status csa_forward(const csa_params* p, csa_dtype io, int32_t B, int32_t T,
                       const csa_forward_args* a, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(a != nullptr, "args is NULL");
  TRY(check_mqa_args(p, io, B, T, a->q, a->q_pos, a->kv_cache, a->N_cap, a->win_kv, a->L_raw,
                     a->win_pos0, a->sink, a->q_rms_w, a->out));
  TRY(check_index_args(p, a->idx_dtype, B, T, a->N_cap, a->qI, a->qI_scale, a->w, a->KI,
                       a->KI_scale, a->q_pos));
  TRY(check_topk(p));
  REQUIRE(p->overlap == 1, "csa_forward is the CSA layer (overlap must be 1)");
  if ((int64_t)B * T == 0) return ok();
  REQUIRE_PTR(a->out_idx);
  OPTIONAL_PTR(a->out_scores);
  const size_t need = csa_workspace_size(p, CSA_WS_FORWARD, a->idx_dtype, B, T, a->N_cap);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws))
    return fail(CSA_ERR_WORKSPACE, "csa_forward needs %zu workspace bytes (got %zu)", need,
                ws_bytes);
  cudaStream_t st = (cudaStream_t)stream;
  if (a->Ca != nullptr) {
    TRY(csa_compress(p, io, B, a->n_tok, a->first_entry, a->N_cap, a->Ca, a->Cb, a->Za, a->Zb,
                     a->bias, a->prev_Cb, a->prev_Zb, a->kv_rms_w, 1, a->kv_cache, stream));
  }
  char* base = static_cast<char*>(ws);
  const size_t sb = scores_bytes(B, T, a->N_cap);
  const size_t tb = round_up(csa::topk_workspace_bytes(B, T, a->N_cap, p->topk));
  float* scores = a->out_scores ? a->out_scores : reinterpret_cast<float*>(base);
  auto ma = make_mqa(p, B, T, a->q, a->q_pos, a->kv_cache, a->N_cap, a->out_idx, p->topk,
                     a->win_kv, a->L_raw, a->win_pos0, a->sink, a->q_rms_w, a->out);
  // the decode selector's last kernel (rank) waited for the filter, which wrote q_hat, so the
  // attention may copy q_hat before its own wait; after the one-kernel row selector, which
  // writes q_hat itself, it is launched the ordinary way
  ma.chained = csa::topk_decode_path(B, T, a->N_cap, p->topk);
  const size_t mb = round_up(csa::mqa_workspace_bytes(ma));
  csa::TopkArgs t{};
  t.B = B; t.T = T; t.m = p->m; t.k = p->topk; t.n_cap = a->N_cap; t.scores = scores;
  t.q_pos = a->q_pos; t.out_idx = a->out_idx;
  if (io == CSA_BF16 && forward_qhat(p, B, T, a->N_cap)) {
    t.qj.q = a->q;
    t.qj.q_rms_w = a->q_rms_w;
    t.qj.qhat = base + sb + tb + mb;
    t.qj.H = p->n_heads;
    t.qj.r = p->rope_dims;
    t.qj.eps = p->rms_eps;
    t.qj.rope_base = p->rope_base;
    for (int i = 0; i < p->rope_dims / 2; ++i)
      t.qj.inv_freq[i] = csa::rope_inv_freq(i, p->rope_dims, (double)p->rope_base);
    ma.qhat = t.qj.qhat;
  }
  TRY(index_then_topk(p, a->idx_dtype, B, T, a->N_cap, a->qI, a->qI_scale, a->w, a->KI,
                      a->KI_scale, a->q_pos, scores, t, base + sb, tb, st));
  TRY(cuda_status(csa::launch_mqa(ma, io == CSA_BF16, base + sb + tb, mb, st), "sparse MQA"));
  return ok();
}

csa_status csa_forward_paged(const csa_params* p, int32_t B, int32_t T, const csa_paged_kv* kv,
                             const csa_paged_kv* keys, int32_t bf16_scores, const void* qI,
                             const void* qI_scale, const float* w, const void* q,
                             const void* q_rms_w,
                             const int64_t* q_pos, const void* win_kv, int64_t L_raw,
                             const int64_t* win_pos0, const float* sink, int32_t* out_idx,
                             void* out_scores, void* out, void* ws, size_t ws_bytes,
                             void* stream) {
  TRY(check_params(p));
  TRY(check_topk(p));
  REQUIRE(p->overlap == 1, "csa_forward_paged is the CSA layer (overlap must be 1)");
  REQUIRE(bf16_scores == 0 || bf16_scores == 1, "bf16_scores must be 0 or 1");
  KvLayout lay;
  int64_t N_cap = 0;
  TRY(paged_layout(kv, &lay, &N_cap));
  TRY(check_paged_keys(keys));
  REQUIRE((int64_t)keys->page_rows * keys->max_pages == N_cap,
          "the KV and key pools must cover the same entries (page_rows * max_pages)");
  if (keys->fmt != CSA_MXFP4) REQUIRE(qI_scale == nullptr, "qI_scale is for MXFP4 queries only");
  TRY(check_mqa_args(p, CSA_BF16, B, T, q, q_pos, kv->pages, N_cap, win_kv, L_raw, win_pos0, sink,
                     q_rms_w, out, true));
  TRY(check_index_args(p, keys->fmt, B, T, N_cap, qI, qI_scale, w, keys->pages, keys->scales,
                       q_pos));
  if ((int64_t)B * T == 0) return ok();
  REQUIRE_PTR(out_idx);
  OPTIONAL_PTR(out_scores);
  TRY(check_paged_index(p, keys, B, T, qI, qI_scale, w, q_pos));
  auto ma = make_mqa(p, B, T, q, q_pos, kv->pages, N_cap, out_idx, p->topk, win_kv, L_raw,
                     win_pos0, sink, q_rms_w, out);
  const bool rope_ok = !lay.mixed ||
                       (p->rope_dims > 0 && p->rope_dims < p->c && p->rope_dims % 16 == 0);
  if (!rope_ok || !csa::mqa_tc_supported(ma, true))
    return fail(CSA_ERR_UNSUPPORTED,
                "csa_forward_paged: needs the tensor-core attention (c = 512, n_heads a multiple "
                "of 64; mixed rows: rope_dims a multiple of 16 in (0, 512))");
  const size_t need = csa_workspace_size(p, CSA_WS_FORWARD, keys->fmt, B, T, N_cap);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws))
    return fail(CSA_ERR_WORKSPACE, "csa_forward_paged needs %zu workspace bytes (got %zu)", need,
                ws_bytes);
  cudaStream_t st = (cudaStream_t)stream;
  char* base = static_cast<char*>(ws);
  const size_t sb = scores_bytes(B, T, N_cap);  // room for fp32 (or bf16) scores
  const size_t tb = round_up(csa::topk_workspace_bytes(B, T, N_cap, p->topk));
  void* sc = out_scores ? out_scores : base;
  ma.kv_scale = lay.mixed ? lay.scales : nullptr;
  ma.page_table = lay.page_table;
  ma.n_pages = lay.n_pages;
  ma.page_rows = lay.page_rows;
  ma.max_pages = lay.max_pages;
  ma.chained = csa::topk_decode_path(B, T, N_cap, p->topk);  // as in csa_forward
  const size_t mb = round_up(csa::mqa_workspace_bytes(ma));
  csa::TopkArgs t{};
  t.B = B; t.T = T; t.m = p->m; t.k = p->topk; t.n_cap = N_cap; t.q_pos = q_pos;
  t.out_idx = out_idx;
  if (bf16_scores) t.scores16 = sc;
  else t.scores = static_cast<float*>(sc);
  if (forward_qhat(p, B, T, N_cap)) {
    t.qj.q = q;
    t.qj.q_rms_w = q_rms_w;
    t.qj.qhat = base + sb + tb + mb;
    t.qj.H = p->n_heads;
    t.qj.r = p->rope_dims;
    t.qj.eps = p->rms_eps;
    t.qj.rope_base = p->rope_base;
    for (int i = 0; i < p->rope_dims / 2; ++i)
      t.qj.inv_freq[i] = csa::rope_inv_freq(i, p->rope_dims, (double)p->rope_base);
    ma.qhat = t.qj.qhat;
  }
  TRY(index_then_topk(p, keys->fmt, B, T, N_cap, qI, qI_scale, w, keys->pages, keys->scales,
                      q_pos, bf16_scores ? nullptr : static_cast<float*>(sc), t, base + sb, tb,
                      st, bf16_scores ? sc : nullptr, keys));
  TRY(cuda_status(csa::launch_mqa(ma, true, base + sb + tb, mb, st), "sparse MQA (paged)"));
  return ok();
}

uint64_t csa_kernel_launches(void) { return csa::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

namespace csa {

csa_status report_error(csa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace csa
