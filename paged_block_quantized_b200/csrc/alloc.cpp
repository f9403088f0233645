// alloc.cpp -- host block allocator: LIFO free list plus per-block reference counts.
//
// deepinsea.top "PagedAttention 内存管理深度解析", section "分页机制设计": blocks needed for a request
// are (num_tokens + block_size - 1) / block_size, allocation fails when too few are free, and
// freeing returns the blocks to the free list. tbr8.org "如何通过 PagedAttention 与分块量化结合..."
// §5 item 3: a pool of physical blocks is set up once and block ids are released through logical
// reference counts. deepinsea.top, section "Copy-on-Write 机制": sequences share blocks and a block
// is copied only when a sharer is about to write to it. Host memory only; not thread-safe.
#include <algorithm>
#include <cstdint>
#include <new>
#include <vector>

#include "../../include/pkv.h"

struct pkv_allocator {
  std::vector<int32_t> free_list;  // top of the stack = back
  std::vector<int32_t> refcount;   // 0 = free
};

extern "C" {

int32_t pkv_blocks_for_tokens(int64_t num_tokens, int32_t block_size) {
  if (num_tokens < 0 || block_size <= 0) return -1;
  const int64_t n = (num_tokens + block_size - 1) / block_size;
  return n > INT32_MAX ? -1 : (int32_t)n;
}

pkv_status pkv_alloc_create(int32_t num_blocks, pkv_allocator** out_handle) {
  if (out_handle == nullptr || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  pkv_allocator* h = new (std::nothrow) pkv_allocator;
  if (h == nullptr) return PKV_ERR_OUT_OF_BLOCKS;
  h->refcount.assign((size_t)num_blocks, 0);
  h->free_list.reserve((size_t)num_blocks);
  // pushed in descending order so that the first blocks handed out are 0, 1, 2, ...
  for (int32_t b = num_blocks - 1; b >= 0; --b) h->free_list.push_back(b);
  *out_handle = h;
  return PKV_OK;
}

void pkv_alloc_destroy(pkv_allocator* h) { delete h; }

int32_t pkv_alloc_num_free(const pkv_allocator* h) { return h ? (int32_t)h->free_list.size() : -1; }

int32_t pkv_alloc_refcount(const pkv_allocator* h, int32_t block_id) {
  if (h == nullptr || block_id < 0 || (size_t)block_id >= h->refcount.size()) return -1;
  return h->refcount[(size_t)block_id];
}

pkv_status pkv_alloc_blocks(pkv_allocator* h, int32_t n, int32_t* ids) {
  if (h == nullptr || n < 0 || (n > 0 && ids == nullptr)) return PKV_ERR_INVALID_ARG;
  if ((size_t)n > h->free_list.size()) return PKV_ERR_OUT_OF_BLOCKS;  // all or nothing
  for (int32_t i = 0; i < n; ++i) {
    const int32_t b = h->free_list.back();
    h->free_list.pop_back();
    h->refcount[(size_t)b] = 1;
    ids[i] = b;
  }
  return PKV_OK;
}

static bool all_allocated(const pkv_allocator* h, const int32_t* ids, int32_t n) {
  for (int32_t i = 0; i < n; ++i) {
    if (ids[i] < 0 || (size_t)ids[i] >= h->refcount.size() || h->refcount[(size_t)ids[i]] <= 0) return false;
  }
  return true;
}

pkv_status pkv_alloc_fork(pkv_allocator* h, const int32_t* ids, int32_t n) {
  if (h == nullptr || n < 0 || (n > 0 && ids == nullptr)) return PKV_ERR_INVALID_ARG;
  if (!all_allocated(h, ids, n)) return PKV_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) ++h->refcount[(size_t)ids[i]];
  return PKV_OK;
}

pkv_status pkv_alloc_release(pkv_allocator* h, const int32_t* ids, int32_t n) {
  if (h == nullptr || n < 0 || (n > 0 && ids == nullptr)) return PKV_ERR_INVALID_ARG;
  // a block listed k times must hold at least k references (checked before anything changes)
  for (int32_t i = 0; i < n; ++i) {
    if (ids[i] < 0 || (size_t)ids[i] >= h->refcount.size()) return PKV_ERR_INVALID_ARG;
  }
  // runs of equal ids in a sorted copy: cost O(n log n) in the ids, independent of the pool size
  std::vector<int32_t> sorted(ids, ids + n);
  std::sort(sorted.begin(), sorted.end());
  for (size_t i = 0; i < sorted.size();) {
    size_t j = i + 1;
    while (j < sorted.size() && sorted[j] == sorted[i]) ++j;
    if ((int64_t)(j - i) > h->refcount[(size_t)sorted[i]]) return PKV_ERR_INVALID_ARG;  // double free
    i = j;
  }
  for (int32_t i = 0; i < n; ++i) {
    int32_t& rc = h->refcount[(size_t)ids[i]];
    if (--rc == 0) h->free_list.push_back(ids[i]);
  }
  return PKV_OK;
}

pkv_status pkv_alloc_cow(pkv_allocator* h, int32_t block_id, int32_t* new_id) {
  if (h == nullptr || new_id == nullptr) return PKV_ERR_INVALID_ARG;
  if (!all_allocated(h, &block_id, 1)) return PKV_ERR_INVALID_ARG;
  int32_t& rc = h->refcount[(size_t)block_id];
  if (rc == 1) {
    *new_id = block_id;
    return PKV_OK;
  }
  if (h->free_list.empty()) return PKV_ERR_OUT_OF_BLOCKS;
  const int32_t b = h->free_list.back();
  h->free_list.pop_back();
  h->refcount[(size_t)b] = 1;
  --rc;
  *new_id = b;
  return PKV_OK;
}

}  // extern "C"
