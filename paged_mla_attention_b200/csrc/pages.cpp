// Host-side page pool for the paged KV cache.
//
// The FlashMLA overview (section 4.2(1)) describes the cache as fixed 64-token
// physical pages handed to sequences through block_table; the pages give no
// allocator.  This one keeps a LIFO free list of page ids plus an ownership
// bit per page, so that a page is never handed out twice and a page that is
// not allocated can not be freed.  Every call is all-or-nothing: on an error
// the pool is unchanged.  Calls are serialised by a mutex.
#include <cstdint>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/pagedmla.h"
#include "pagedmla_internal.cuh"

struct pmla_page_pool {
  std::mutex mu;
  std::vector<int32_t> free_list;  // stack of free page ids
  std::vector<uint8_t> in_use;     // 1 while a page is allocated
};

namespace {

constexpr int kPage = PMLA_PAGE_SIZE;

int pages_for(long long len) { return (int)((len + kPage - 1) / kPage); }

// Requires the pool's mutex.  True when all n ids are allocated and distinct;
// the pool is left as it was either way.
bool all_allocated_distinct(pmla_page_pool* p, int n, const int32_t* pages) {
  bool ok = true;
  int marked = 0;
  for (; marked < n; ++marked) {
    const int32_t id = pages[marked];
    if (id < 0 || id >= (int32_t)p->in_use.size() || p->in_use[id] != 1) {  // free, bad, or repeated
      ok = false;
      break;
    }
    p->in_use[id] = 2;  // seen in this call
  }
  for (int i = 0; i < marked; ++i) p->in_use[pages[i]] = 1;
  return ok;
}

}  // namespace

extern "C" {

PMLA_API int pmla_page_pool_create(int num_pages, pmla_page_pool** out) {
  if (!out || num_pages < 1) return PMLA_ERR_INVALID_ARG;
  pmla_page_pool* p = new (std::nothrow) pmla_page_pool;
  if (!p) return PMLA_ERR_INVALID_ARG;
  p->free_list.resize(num_pages);
  p->in_use.assign(num_pages, 0);
  // the stack pops the lowest ids first
  for (int i = 0; i < num_pages; ++i) p->free_list[i] = num_pages - 1 - i;
  *out = p;
  return PMLA_OK;
}

PMLA_API void pmla_page_pool_destroy(pmla_page_pool* pool) { delete pool; }

PMLA_API int pmla_page_pool_num_free(pmla_page_pool* pool) {
  if (!pool) return PMLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(pool->mu);
  return (int)pool->free_list.size();
}

PMLA_API int pmla_page_pool_alloc(pmla_page_pool* pool, int n, int32_t* pages_out) {
  if (!pool || n < 0 || (n > 0 && !pages_out)) return PMLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(pool->mu);
  if ((size_t)n > pool->free_list.size()) {
    pmla::set_last_error("page pool exhausted");
    return PMLA_ERR_EXHAUSTED;
  }
  for (int i = 0; i < n; ++i) {
    const int32_t id = pool->free_list.back();
    pool->free_list.pop_back();
    pool->in_use[id] = 1;
    pages_out[i] = id;
  }
  return PMLA_OK;
}

PMLA_API int pmla_page_pool_free(pmla_page_pool* pool, int n, const int32_t* pages) {
  if (!pool || n < 0 || (n > 0 && !pages)) return PMLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(pool->mu);
  if (!all_allocated_distinct(pool, n, pages)) {
    pmla::set_last_error("page id out of range, not allocated, or repeated");
    return PMLA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n; ++i) {
    pool->in_use[pages[i]] = 0;
    pool->free_list.push_back(pages[i]);
  }
  return PMLA_OK;
}

PMLA_API int pmla_page_pool_grow_sequence(pmla_page_pool* pool, int32_t* block_table_row,
                                          int max_pages, int cur_len, int new_len) {
  if (!pool || !block_table_row || max_pages < 1 || cur_len < 0 || new_len < cur_len)
    return PMLA_ERR_INVALID_ARG;
  const int have = pages_for(cur_len), want = pages_for(new_len);
  if (want > max_pages) {
    pmla::set_last_error("sequence length past the block-table row");
    return PMLA_ERR_INVALID_ARG;
  }
  if (want == have) return PMLA_OK;
  return pmla_page_pool_alloc(pool, want - have, block_table_row + have);
}

PMLA_API int pmla_page_pool_release_sequence(pmla_page_pool* pool, const int32_t* block_table_row,
                                             int len) {
  if (!pool || len < 0 || (len > 0 && !block_table_row)) return PMLA_ERR_INVALID_ARG;
  return pmla_page_pool_free(pool, pages_for(len), block_table_row);
}

}  // extern "C"
