// Host-side page allocator of the state cache's page pools.
//
// 【论文解读】DeepSeek-V4, 二、基础设施 (六) 推理框架: the finished compressed entries live in a
// classical cache whose blocks cover a multiple of lcm(m, m') raw tokens. DeepseekV4论文解析,
// 2. Hybrid Attention：CSA + HCA (从注意力公式到可部署系统): one logical block of 128 raw
// tokens holds 32 CSA entries or 1 HCA entry, kept in a paged cache. A layer's requests
// share one pool of physical pages; each request's row of the page table maps its logical
// pages to physical ones. The decode kernels read that table (csa_state_append writes a
// finished entry through it, the paged attention and indexers read through it); this file
// only decides which physical page backs which logical page.
//
// Free pages form a FIFO: the pool starts as 0 .. n_pages-1 and a released request's
// pages join the back in logical order, so a page just given back is the last to be reused.
#include <cstdint>
#include <cstdio>
#include <deque>
#include <new>
#include <vector>

#include "csa.h"
#include "internal.h"

struct csa_page_alloc {
  int32_t n_pages, B, max_pages;
  std::deque<int32_t> free_list;
  std::vector<int32_t> table;   // [B, max_pages], -1 = not mapped
  std::vector<int32_t> mapped;  // [B]: logical pages 0 .. mapped[b]-1 are mapped
};

extern "C" {

csa_status csa_page_alloc_create(int32_t n_pages, int32_t B, int32_t max_pages,
                                 csa_page_alloc** out) {
  if (out == nullptr) return csa::report_error(CSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (n_pages < 1 || B < 1 || max_pages < 1)
    return csa::report_error(CSA_ERR_INVALID_ARG,
                             "n_pages, B and max_pages must be >= 1 (got %d, %d, %d)", n_pages,
                             B, max_pages);
  if ((int64_t)B * max_pages > (int64_t)1 << 30)
    return csa::report_error(CSA_ERR_INVALID_ARG, "B * max_pages too large");
  csa_page_alloc* a = new (std::nothrow) csa_page_alloc();
  if (a == nullptr) return csa::report_error(CSA_ERR_INVALID_ARG, "host allocation failed");
  a->n_pages = n_pages;
  a->B = B;
  a->max_pages = max_pages;
  for (int32_t p = 0; p < n_pages; ++p) a->free_list.push_back(p);
  a->table.assign((size_t)B * max_pages, -1);
  a->mapped.assign((size_t)B, 0);
  *out = a;
  return csa::report_error(CSA_OK, "");
}

void csa_page_alloc_destroy(csa_page_alloc* a) { delete a; }

csa_status csa_page_alloc_reserve(csa_page_alloc* a, int32_t b, int32_t n_logical) {
  if (a == nullptr) return csa::report_error(CSA_ERR_INVALID_ARG, "allocator is NULL");
  if (b < 0 || b >= a->B)
    return csa::report_error(CSA_ERR_INVALID_ARG, "request %d outside [0, %d)", b, a->B);
  if (n_logical < 0 || n_logical > a->max_pages)
    return csa::report_error(CSA_ERR_INVALID_ARG, "n_logical %d outside [0, %d]", n_logical,
                             a->max_pages);
  const int32_t have = a->mapped[b];
  if (n_logical <= have) return csa::report_error(CSA_OK, "");
  const int32_t need = n_logical - have;
  if ((size_t)need > a->free_list.size())
    return csa::report_error(CSA_ERR_NO_PAGES, "request %d needs %d more pages, %zu free", b,
                             need, a->free_list.size());
  int32_t* row = a->table.data() + (size_t)b * a->max_pages;
  for (int32_t k = have; k < n_logical; ++k) {
    row[k] = a->free_list.front();
    a->free_list.pop_front();
  }
  a->mapped[b] = n_logical;
  return csa::report_error(CSA_OK, "");
}

csa_status csa_page_alloc_release(csa_page_alloc* a, int32_t b) {
  if (a == nullptr) return csa::report_error(CSA_ERR_INVALID_ARG, "allocator is NULL");
  if (b < 0 || b >= a->B)
    return csa::report_error(CSA_ERR_INVALID_ARG, "request %d outside [0, %d)", b, a->B);
  int32_t* row = a->table.data() + (size_t)b * a->max_pages;
  for (int32_t k = 0; k < a->mapped[b]; ++k) {
    a->free_list.push_back(row[k]);
    row[k] = -1;
  }
  a->mapped[b] = 0;
  return csa::report_error(CSA_OK, "");
}

const int32_t* csa_page_alloc_table(const csa_page_alloc* a) {
  return a == nullptr ? nullptr : a->table.data();
}

int32_t csa_page_alloc_free_pages(const csa_page_alloc* a) {
  return a == nullptr ? -1 : (int32_t)a->free_list.size();
}

int32_t csa_page_alloc_mapped(const csa_page_alloc* a, int32_t b) {
  return (a == nullptr || b < 0 || b >= a->B) ? -1 : a->mapped[b];
}

int32_t csa_state_pages_needed(int32_t m, int32_t page_rows, int64_t n_tok) {
  if (m < 1 || page_rows < 1 || n_tok < 0) return -1;
  const int64_t entries = n_tok / m;
  const int64_t pages = (entries + page_rows - 1) / page_rows;
  return pages > INT32_MAX ? -1 : (int32_t)pages;
}

}  // extern "C"
