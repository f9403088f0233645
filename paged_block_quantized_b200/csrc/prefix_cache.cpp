// prefix_cache.cpp -- automatic prefix caching: an index from token blocks to physical blocks.
//
// yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section "Prefix Caching与多轮对话场景
// 优化实践": when a request arrives, the pool is searched for blocks that already hold a matching
// prefix; on a hit the request maps its table straight onto those physical blocks and only its
// new tokens need computing. Section "PagedAttention分页注意力机制与vLLM实现": requests with the same
// prefix share physical blocks. deepinsea.top "PagedAttention 内存管理深度解析", "Copy-on-Write 机制":
// shared blocks are copied only when a sharer writes into one.
//
// What is cached: whole blocks only (a partly filled block is still being written). A block is
// identified by its own token ids together with everything before it, so an entry is the pair
// (parent entry, the block's block_size token ids); lookups hash that pair and then compare it
// exactly, so a hash collision can never produce a false hit. The cache holds one reference
// (through the pool's pkv_allocator) on every block it indexes; a block that only the cache
// references is evictable, least recently used first, and evicting it drops its descendants
// from the index too (they can no longer be reached from the root). Host memory only; not
// thread-safe; the allocator must outlive the cache.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pkv.h"

namespace {

struct Entry {
  int32_t parent;                  // entry index, -1 for a first block
  int32_t block_id;                // physical block
  uint64_t hash;
  uint64_t last_use;               // tick of the last match or insert
  std::vector<int32_t> tokens;     // the block's token ids
  std::vector<int32_t> children;   // entry indices
  bool live;
};

// 64-bit mix of (parent hash, tokens): splitmix64 finalizer over a running state.
uint64_t mix(uint64_t x) {
  x += 0x9e3779b97f4a7c15ull;
  x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
  x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}
uint64_t block_hash(uint64_t parent_hash, const int32_t* tokens, int32_t n) {
  uint64_t h = mix(parent_hash ^ 0x5bd1e995ull);
  for (int32_t i = 0; i < n; ++i) h = mix(h ^ (uint32_t)tokens[i]);
  return h;
}

}  // namespace

struct pkv_prefix_cache {
  pkv_allocator* alloc;
  int32_t block_size;
  uint64_t tick;
  std::vector<Entry> entries;
  std::vector<int32_t> free_entries;
  std::unordered_multimap<uint64_t, int32_t> index;  // hash -> entry
  std::vector<int32_t> roots;                        // entries without a parent

  int32_t find(int32_t parent, const int32_t* tokens) const {
    const uint64_t ph = parent < 0 ? 0 : entries[(size_t)parent].hash;
    const uint64_t h = block_hash(ph, tokens, block_size);
    auto range = index.equal_range(h);
    for (auto it = range.first; it != range.second; ++it) {
      const Entry& e = entries[(size_t)it->second];
      if (e.live && e.parent == parent && std::memcmp(e.tokens.data(), tokens, sizeof(int32_t) * block_size) == 0)
        return it->second;
    }
    return -1;
  }

  // drop entry i and its descendants from the index, releasing the cache's reference on each block
  void drop(int32_t i) {
    std::vector<int32_t> stack{i};
    // detach from the parent (or the roots)
    const int32_t par = entries[(size_t)i].parent;
    std::vector<int32_t>& sib = par < 0 ? roots : entries[(size_t)par].children;
    sib.erase(std::remove(sib.begin(), sib.end(), i), sib.end());
    while (!stack.empty()) {
      const int32_t j = stack.back();
      stack.pop_back();
      Entry& e = entries[(size_t)j];
      for (int32_t c : e.children) stack.push_back(c);
      auto range = index.equal_range(e.hash);
      for (auto it = range.first; it != range.second; ++it) {
        if (it->second == j) {
          index.erase(it);
          break;
        }
      }
      (void)pkv_alloc_release(alloc, &e.block_id, 1);
      e.live = false;
      e.children.clear();
      e.tokens.clear();
      free_entries.push_back(j);
    }
  }
};

extern "C" {

pkv_status pkv_prefix_cache_create(pkv_allocator* alloc, int32_t block_size, pkv_prefix_cache** out) {
  if (alloc == nullptr || out == nullptr || block_size <= 0) return PKV_ERR_INVALID_ARG;
  pkv_prefix_cache* pc = new (std::nothrow) pkv_prefix_cache;
  if (pc == nullptr) return PKV_ERR_OUT_OF_BLOCKS;
  pc->alloc = alloc;
  pc->block_size = block_size;
  pc->tick = 0;
  *out = pc;
  return PKV_OK;
}

void pkv_prefix_cache_destroy(pkv_prefix_cache* pc) {
  if (pc == nullptr) return;
  while (!pc->roots.empty()) pc->drop(pc->roots.back());
  delete pc;
}

int32_t pkv_prefix_cache_size(const pkv_prefix_cache* pc) {
  return pc ? (int32_t)(pc->entries.size() - pc->free_entries.size()) : -1;
}

int32_t pkv_prefix_cache_evictable(const pkv_prefix_cache* pc) {
  if (pc == nullptr) return -1;
  int32_t n = 0;
  for (const Entry& e : pc->entries)
    if (e.live && pkv_alloc_refcount(pc->alloc, e.block_id) == 1) ++n;
  return n;
}

pkv_status pkv_prefix_match(pkv_prefix_cache* pc, const int32_t* tokens, int64_t n_tokens, int32_t* block_ids,
                            int32_t max_blocks, int32_t* n_matched) {
  if (pc == nullptr || n_matched == nullptr || n_tokens < 0 || max_blocks < 0) return PKV_ERR_INVALID_ARG;
  if ((n_tokens > 0 && tokens == nullptr) || (max_blocks > 0 && block_ids == nullptr)) return PKV_ERR_INVALID_ARG;
  const int64_t full = n_tokens / pc->block_size;
  std::vector<int32_t> hit;
  int32_t parent = -1;
  for (int64_t i = 0; i < full && (int64_t)hit.size() < max_blocks; ++i) {
    const int32_t e = pc->find(parent, tokens + i * pc->block_size);
    if (e < 0) break;
    hit.push_back(e);
    parent = e;
  }
  // every hit gains one reference for the caller (blocks the cache holds are allocated)
  std::vector<int32_t> ids(hit.size());
  for (size_t i = 0; i < hit.size(); ++i) ids[i] = pc->entries[(size_t)hit[i]].block_id;
  if (!ids.empty()) {
    const pkv_status st = pkv_alloc_fork(pc->alloc, ids.data(), (int32_t)ids.size());
    if (st != PKV_OK) return st;
  }
  ++pc->tick;
  for (size_t i = 0; i < hit.size(); ++i) {
    pc->entries[(size_t)hit[i]].last_use = pc->tick;
    block_ids[i] = ids[i];
  }
  *n_matched = (int32_t)hit.size();
  return PKV_OK;
}

pkv_status pkv_prefix_insert(pkv_prefix_cache* pc, const int32_t* tokens, int64_t n_tokens, const int32_t* block_ids,
                             int32_t n_blocks) {
  if (pc == nullptr || n_tokens < 0 || n_blocks < 0) return PKV_ERR_INVALID_ARG;
  if ((n_tokens > 0 && tokens == nullptr) || (n_blocks > 0 && block_ids == nullptr)) return PKV_ERR_INVALID_ARG;
  const int64_t full = std::min<int64_t>(n_tokens / pc->block_size, n_blocks);
  // every block to be registered must be allocated (checked before anything changes)
  for (int64_t i = 0; i < full; ++i)
    if (pkv_alloc_refcount(pc->alloc, block_ids[i]) <= 0) return PKV_ERR_INVALID_ARG;
  ++pc->tick;
  int32_t parent = -1;
  for (int64_t i = 0; i < full; ++i) {
    const int32_t* tk = tokens + i * pc->block_size;
    int32_t e = pc->find(parent, tk);
    if (e < 0) {
      // a new entry: the cache takes a reference on the caller's block
      const pkv_status st = pkv_alloc_fork(pc->alloc, &block_ids[i], 1);
      if (st != PKV_OK) return st;
      if (!pc->free_entries.empty()) {
        e = pc->free_entries.back();
        pc->free_entries.pop_back();
      } else {
        e = (int32_t)pc->entries.size();
        pc->entries.emplace_back();
      }
      Entry& en = pc->entries[(size_t)e];
      en.parent = parent;
      en.block_id = block_ids[i];
      en.hash = block_hash(parent < 0 ? 0 : pc->entries[(size_t)parent].hash, tk, pc->block_size);
      en.tokens.assign(tk, tk + pc->block_size);
      en.children.clear();
      en.live = true;
      pc->index.emplace(en.hash, e);
      if (parent < 0) pc->roots.push_back(e);
      else pc->entries[(size_t)parent].children.push_back(e);
    }
    pc->entries[(size_t)e].last_use = pc->tick;
    parent = e;
  }
  return PKV_OK;
}

pkv_status pkv_prefix_alloc(pkv_prefix_cache* pc, int32_t n, int32_t* ids) {
  if (pc == nullptr || n < 0 || (n > 0 && ids == nullptr)) return PKV_ERR_INVALID_ARG;
  // all or nothing: each evictable entry (only the cache references its block) frees one block
  if (pkv_alloc_num_free(pc->alloc) + pkv_prefix_cache_evictable(pc) < n) return PKV_ERR_OUT_OF_BLOCKS;
  // evict least recently used blocks that only the cache references until n blocks are free
  while (pkv_alloc_num_free(pc->alloc) < n) {
    int32_t victim = -1;
    for (size_t i = 0; i < pc->entries.size(); ++i) {
      const Entry& e = pc->entries[i];
      if (!e.live || pkv_alloc_refcount(pc->alloc, e.block_id) != 1) continue;
      if (victim < 0 || e.last_use < pc->entries[(size_t)victim].last_use) victim = (int32_t)i;
    }
    if (victim < 0) return PKV_ERR_OUT_OF_BLOCKS;  // not reached: the count above covers n
    pc->drop(victim);
  }
  return pkv_alloc_blocks(pc->alloc, n, ids);
}

}  // extern "C"
