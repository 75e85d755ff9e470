// Host build of the state-append arithmetic (csrc/state_append.cuh) for the CPU tests: the
// same __host__ __device__ functions the kernel calls, run request by request and channel
// by channel in the kernel's order, on host arrays. Every offset written is checked against
// the buffer sizes first. Test infrastructure: the library never links it.
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <vector>

#include "state_append.cuh"

namespace {

template <typename T>
int run(csa::state::Args a, int32_t* status, size_t state_elems, size_t ring_elems,
        size_t page_elems) {
  using namespace csa::state;
  std::vector<float> row(a.c);
  for (int b = 0; b < a.B; ++b) {
    const int64_t t = a.pos[b];
    int64_t i = 0;
    size_t off = 0;
    const int s = append_status(a, b, t, &i, &off);
    status[b] = s;
    if (s < 0) continue;
    for (int j = 0; j < a.c; ++j) {
      for (int r = 0; r < rows(a); ++r)
        if (state_index(a, b, t, r, j) >= state_elems) return -10;
      if (a.win_ring && ((size_t)b * a.n_win + (size_t)(t % a.n_win)) * a.c + j >= ring_elems)
        return -11;
      store_channel<T>(a, b, t, j);
    }
    if (s == kAppendOnly) continue;
    if (off + (size_t)a.c > page_elems) return -12;
    float ssf = 0.f;
    for (int j = 0; j < a.c; ++j) {
      row[j] = pool_channel<T>(a, b, i, j);
      ssf = fmaf(row[j], row[j], ssf);
    }
    T* out = static_cast<T*>(a.pages) + off;
    if (!a.finalize) {
      for (int j = 0; j < a.c; ++j) st(out, j, row[j]);
      continue;
    }
    const float rstd = 1.f / sqrtf(ssf / (float)a.c + a.eps);
    for (int j = 0; j < a.c; ++j) st(out, j, final_channel<T>(a, row.data(), rstd, i, j));
  }
  return 0;
}

}  // namespace

extern "C" int state_append_host(int bf16, int B, int m, int c, int overlap, int rope_dims,
                                 double rope_base, int finalize, int n_win, int n_pages,
                                 int page_rows, int max_pages, float eps, const int64_t* pos,
                                 const void* Ca, const void* Cb, const void* Za, const void* Zb,
                                 const void* win_row, const void* bias, const void* rms_w,
                                 void* state, void* win_ring, void* pages,
                                 const int32_t* page_table, int32_t* status) {
  csa::state::Args a{};
  a.B = B; a.m = m; a.c = c; a.overlap = overlap; a.rope_dims = rope_dims;
  a.finalize = finalize; a.n_win = n_win; a.n_pages = n_pages; a.page_rows = page_rows;
  a.max_pages = max_pages; a.eps = eps; a.pos = pos; a.Ca = Ca; a.Cb = Cb; a.Za = Za;
  a.Zb = Zb; a.win_row = win_row; a.bias = bias; a.rms_w = rms_w; a.state = state;
  a.win_ring = win_ring; a.pages = pages; a.page_table = page_table;
  for (int p = 0; p < rope_dims / 2; ++p)
    a.inv_freq[p] = std::exp2(-2.0 * p / rope_dims * std::log2(rope_base));
  const size_t state_elems = (size_t)B * (overlap ? 2 * m : m) * (overlap ? 4 : 2) * c;
  const size_t ring_elems = (size_t)B * (n_win > 0 ? n_win : 0) * c;
  const size_t page_elems = (size_t)n_pages * page_rows * c;
  return bf16 ? run<__nv_bfloat16>(a, status, state_elems, ring_elems, page_elems)
              : run<float>(a, status, state_elems, ring_elems, page_elems);
}
