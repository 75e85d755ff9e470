// csa_topk_noalloc: the stage-3 selector with library-owned scratch.
//
// The selector for few long rows (per-row histograms, counters, lists of sure and boundary
// candidates) needs device scratch, which csa_topk takes from its caller. Some callers have
// none to give: a C or C++ host program that links libcsa directly and has no device
// allocator of its own, or a serving loop that has already reserved the device memory for
// its caches, so that a fresh cudaMalloc would fail or would synchronise the device in the
// middle of a step. For them this entry point takes the scratch from one file-scope
// __device__ array (one copy per device, loaded with the module) and allocates nothing.
//
// Set-up: the first call on a device looks up the array's device address with
// cudaGetSymbolAddress, with that device current, and caches it; make that first call
// before any stream capture. Sharing: every call on a device uses the same array. The
// histograms and counters at its start must be zero when the selector starts, and each call
// zeroes them itself (an asynchronous memset on the call's stream); the candidate lists are
// written before they are read. Two calls whose execution overlaps (different streams, or
// host threads on one device) therefore race on the array: serialise them on one stream.
// The paper defines no such interface; it is plumbing for the selector of 一(三)1(2).
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = CSA_TOPK_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_topk_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];  // per device ordinal, filled on the first call there

cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_topk_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = addr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" csa_status csa_topk_noalloc(const csa_params* p, int32_t B, int32_t T,
                                       int64_t N_cap, const float* scores,
                                       const int64_t* q_pos, int32_t* out_idx, void* stream) {
  // Arguments that csa_topk would reject are passed on to it unchanged (no scratch), so that
  // it reports them with its own message; the size limit is checked on sound sizes only.
  const bool sizes_ok = p != nullptr && p->topk >= 1 && p->topk <= csa::kMaxTopk && B >= 0 &&
                        T >= 0 && N_cap >= 0 && N_cap <= INT32_MAX &&
                        (int64_t)B * T <= 65535 * 64;
  if (!sizes_ok) return csa_topk(p, B, T, N_cap, scores, q_pos, out_idx, nullptr, 0, stream);
  const size_t need = csa::topk_workspace_bytes(B, T, N_cap, p->topk);
  if (need > kScratchBytes)
    return csa::report_error(CSA_ERR_WORKSPACE,
                             "csa_topk_noalloc: B*T=%lld rows of N_cap=%lld with k=%d need %zu "
                             "scratch bytes; the library-owned array holds %zu (use csa_topk "
                             "with caller scratch)",
                             (long long)B * T, (long long)N_cap, p->topk, need, kScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
      return csa::report_error(CSA_ERR_CUDA, "csa_topk_noalloc: scratch address: %s",
                               cudaGetErrorString(e));
  }
  return csa_topk(p, B, T, N_cap, scores, q_pos, out_idx, scratch, need > 0 ? kScratchBytes : 0,
                  stream);
}
