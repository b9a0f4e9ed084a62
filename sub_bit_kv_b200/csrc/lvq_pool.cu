// Host bookkeeping of a page pool (pool mode of lvq_config): which physical page ids are
// handed out to requests.  "LoopVQ summary", section "premises and limits": the cache is
// built from 8-token pages; requests of any length take pages from one shared pool as their
// coded region grows and give them back when they end.
//
// Free ids are kept in an ordered set and handed out lowest first, so that the pages of a
// request tend to form runs of consecutive ids, which the decode copies with one bulk copy
// each.  Host memory only: the device pools and the page table are the caller's buffers.
#include <set>
#include <vector>

#include "lvq_common.cuh"

struct lvq_pool {
  int32_t n_pages;
  std::set<int32_t> free_ids;
};

extern "C" {

lvq_status lvq_pool_create(int32_t n_pages, lvq_pool** out) {
  if (!out || n_pages < 1) return LVQ_EINVAL;
  lvq_pool* p = new (std::nothrow) lvq_pool;
  if (!p) return LVQ_ECAPACITY;
  p->n_pages = n_pages;
  for (int32_t i = 0; i < n_pages; ++i) p->free_ids.insert(p->free_ids.end(), i);
  *out = p;
  return LVQ_OK;
}

void lvq_pool_destroy(lvq_pool* pool) { delete pool; }

lvq_status lvq_pool_alloc(lvq_pool* pool, int32_t n, int32_t* ids) {
  if (!pool || n < 0 || (n > 0 && !ids)) return LVQ_EINVAL;
  if ((size_t)n > pool->free_ids.size()) return LVQ_ECAPACITY;
  for (int32_t i = 0; i < n; ++i) {
    auto it = pool->free_ids.begin();
    ids[i] = *it;
    pool->free_ids.erase(it);
  }
  return LVQ_OK;
}

lvq_status lvq_pool_free(lvq_pool* pool, const int32_t* ids, int32_t n) {
  if (!pool || n < 0 || (n > 0 && !ids)) return LVQ_EINVAL;
  // all or nothing: every id in range, currently handed out, and not repeated
  std::set<int32_t> seen;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = ids[i];
    if (id < 0 || id >= pool->n_pages || pool->free_ids.count(id) || !seen.insert(id).second) return LVQ_EINVAL;
  }
  for (int32_t i = 0; i < n; ++i) pool->free_ids.insert(ids[i]);
  return LVQ_OK;
}

int32_t lvq_pool_available(const lvq_pool* pool) { return pool ? (int32_t)pool->free_ids.size() : -1; }

}  // extern "C"
