// pool.cpp -- host block-pool allocator, prefix cache and slot-mapping helper.
//
// "vLLM" glossary, "PagedAttention": the KV cache is held in fixed-size blocks
// mapped from logical to physical ids and shared across sequences (beam search,
// parallel sampling); "Continuous batching": finished sequences return their
// blocks to the pool; "Prefix caching" / "Automatic prefix caching": a request
// whose prompt starts like an earlier one reuses that request's KV blocks.
// "vLLM v0.7.2" field report, "Field Observations": block pool exhaustion.
// Every operation is O(1) per block id and all-or-nothing.
//
// Prefix cache. Only full blocks are cached (a partial block is still being
// appended to). A cached block is keyed by its 16 token ids and the serial
// number of the cached block before it in the prompt (0 for the first block).
// Serials are never reused, so a key names the whole prefix exactly: neither a
// hash collision nor a block id reused after eviction can hand out a block
// whose contents belong to another prefix (the children of an evicted block
// become unreachable and are evicted in their turn). A
// cached block that no sequence references stays cached ("evictable") until
// the pool needs it: allocation takes truly free ids first, then evicts the
// least recently released evictable block.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pqkv.h"

namespace {

struct PrefixKey {
  uint64_t parent;  // serial of the previous block's cache entry, 0 = none
  int32_t tok[PQKV_BLOCK_SIZE];
  bool operator==(const PrefixKey& o) const {
    return parent == o.parent && std::memcmp(tok, o.tok, sizeof(tok)) == 0;
  }
};

struct PrefixKeyHash {
  size_t operator()(const PrefixKey& k) const {
    // FNV-1a over the key's bytes, then a 64-bit finalizer (splitmix64)
    uint64_t h = 1469598103934665603ull;
    auto mix = [&](uint32_t v) {
      for (int i = 0; i < 4; ++i) {
        h ^= (v >> (8 * i)) & 0xFFu;
        h *= 1099511628211ull;
      }
    };
    mix((uint32_t)k.parent);
    mix((uint32_t)(k.parent >> 32));
    for (int i = 0; i < PQKV_BLOCK_SIZE; ++i) mix((uint32_t)k.tok[i]);
    h ^= h >> 30;
    h *= 0xbf58476d1ce4e5b9ull;
    h ^= h >> 27;
    h *= 0x94d049bb133111ebull;
    h ^= h >> 31;
    return (size_t)h;
  }
};

}  // namespace

struct pqkv_pool {
  int32_t num_blocks;
  std::vector<int32_t> free_ids;  // stack; back() is handed out next
  std::vector<int32_t> refs;
  // prefix cache
  std::unordered_map<PrefixKey, int32_t, PrefixKeyHash> map;
  std::vector<PrefixKey> key;     // key of a cached block
  std::vector<uint64_t> serial;   // serial of a cached block's entry
  std::vector<uint8_t> cached;
  uint64_t next_serial = 1;
  // evictable (cached, no references) blocks: doubly linked list, head = oldest
  std::vector<int32_t> prev, next;
  int32_t head = -1, tail = -1;
  int32_t n_evictable = 0;

  void evictable_push(int32_t id) {
    prev[(size_t)id] = tail;
    next[(size_t)id] = -1;
    if (tail >= 0) next[(size_t)tail] = id; else head = id;
    tail = id;
    ++n_evictable;
  }
  void evictable_remove(int32_t id) {
    const int32_t a = prev[(size_t)id], b = next[(size_t)id];
    if (a >= 0) next[(size_t)a] = b; else head = b;
    if (b >= 0) prev[(size_t)b] = a; else tail = a;
    prev[(size_t)id] = next[(size_t)id] = -1;
    --n_evictable;
  }
  void uncache(int32_t id) {
    map.erase(key[(size_t)id]);
    cached[(size_t)id] = 0;
    serial[(size_t)id] = 0;
  }
  // one id for a new sequence reference (caller checked availability)
  int32_t take() {
    int32_t id;
    if (!free_ids.empty()) {
      id = free_ids.back();
      free_ids.pop_back();
    } else {
      id = head;
      evictable_remove(id);
      uncache(id);
    }
    refs[(size_t)id] = 1;
    return id;
  }
  // a block whose last reference was dropped
  void release(int32_t id) {
    if (cached[(size_t)id]) evictable_push(id); else free_ids.push_back(id);
  }
};

extern "C" {

int pqkv_pool_create(int32_t num_blocks, pqkv_pool** out_pool) {
  if (!out_pool || num_blocks < 1) return PQKV_ERR_ARG;
  pqkv_pool* p = new (std::nothrow) pqkv_pool;
  if (!p) return PQKV_ERR_OOM;
  try {
    p->num_blocks = num_blocks;
    p->refs.assign((size_t)num_blocks, 0);
    p->key.resize((size_t)num_blocks);
    p->serial.assign((size_t)num_blocks, 0);
    p->cached.assign((size_t)num_blocks, 0);
    p->prev.assign((size_t)num_blocks, -1);
    p->next.assign((size_t)num_blocks, -1);
    p->free_ids.resize((size_t)num_blocks);
    for (int32_t i = 0; i < num_blocks; ++i) p->free_ids[(size_t)i] = num_blocks - 1 - i;
  } catch (...) {
    delete p;
    return PQKV_ERR_OOM;
  }
  *out_pool = p;
  return PQKV_OK;
}

void pqkv_pool_destroy(pqkv_pool* pool) { delete pool; }

int pqkv_pool_alloc(pqkv_pool* pool, int n, int32_t* ids_out) {
  if (!pool || n < 0 || (n > 0 && !ids_out)) return PQKV_ERR_ARG;
  if ((size_t)n > pool->free_ids.size() + (size_t)pool->n_evictable) return PQKV_ERR_OOM;
  for (int i = 0; i < n; ++i) ids_out[i] = pool->take();
  return PQKV_OK;
}

int pqkv_pool_share(pqkv_pool* pool, const int32_t* ids, int n) {
  if (!pool || n < 0 || (n > 0 && !ids)) return PQKV_ERR_ARG;
  for (int i = 0; i < n; ++i) {
    if (ids[i] < 0 || ids[i] >= pool->num_blocks) return PQKV_ERR_ARG;
    if (pool->refs[(size_t)ids[i]] <= 0) return PQKV_ERR_STATE;
  }
  for (int i = 0; i < n; ++i) ++pool->refs[(size_t)ids[i]];
  return PQKV_OK;
}

int pqkv_pool_free(pqkv_pool* pool, const int32_t* ids, int n) {
  if (!pool || n < 0 || (n > 0 && !ids)) return PQKV_ERR_ARG;
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= pool->num_blocks) return PQKV_ERR_ARG;
  // drop references, undoing everything if some id runs out of them
  for (int i = 0; i < n; ++i) {
    int32_t& r = pool->refs[(size_t)ids[i]];
    if (r <= 0) {
      for (int k = i - 1; k >= 0; --k) ++pool->refs[(size_t)ids[k]];
      return PQKV_ERR_STATE;
    }
    --r;
  }
  // return blocks that reached zero, each once even if repeated in ids
  for (int i = 0; i < n; ++i) {
    int32_t& r = pool->refs[(size_t)ids[i]];
    if (r == 0) {
      pool->release(ids[i]);
      r = INT_MIN;
    }
  }
  for (int i = 0; i < n; ++i) {
    int32_t& r = pool->refs[(size_t)ids[i]];
    if (r == INT_MIN) r = 0;
  }
  return PQKV_OK;
}

int32_t pqkv_pool_num_free(const pqkv_pool* pool) { return pool ? (int32_t)pool->free_ids.size() : -1; }

int32_t pqkv_pool_num_evictable(const pqkv_pool* pool) { return pool ? pool->n_evictable : -1; }

int32_t pqkv_pool_num_cached(const pqkv_pool* pool) { return pool ? (int32_t)pool->map.size() : -1; }

int pqkv_pool_prefix_lookup(pqkv_pool* pool, const int32_t* token_ids, int num_tokens, int32_t* ids_out,
                            int* num_hit) {
  if (!pool || num_tokens < 0 || (num_tokens > 0 && (!token_ids || !ids_out)) || !num_hit) return PQKV_ERR_ARG;
  int hit = 0;
  PrefixKey k;
  k.parent = 0;
  for (int b = 0; b < num_tokens / PQKV_BLOCK_SIZE; ++b) {
    std::memcpy(k.tok, token_ids + (size_t)b * PQKV_BLOCK_SIZE, sizeof(k.tok));
    const auto it = pool->map.find(k);
    if (it == pool->map.end()) break;
    const int32_t id = it->second;
    if (pool->refs[(size_t)id] == 0) pool->evictable_remove(id);
    ++pool->refs[(size_t)id];
    ids_out[hit++] = id;
    k.parent = pool->serial[(size_t)id];
  }
  *num_hit = hit;
  return PQKV_OK;
}

int pqkv_pool_prefix_insert(pqkv_pool* pool, const int32_t* token_ids, int num_tokens, const int32_t* ids,
                            int num_ids) {
  if (!pool || num_tokens < 0 || num_ids < 0) return PQKV_ERR_ARG;
  const int nfull = std::min(num_tokens / PQKV_BLOCK_SIZE, num_ids);
  if (nfull > 0 && (!token_ids || !ids)) return PQKV_ERR_ARG;
  for (int b = 0; b < nfull; ++b) {
    if (ids[b] < 0 || ids[b] >= pool->num_blocks) return PQKV_ERR_ARG;
    if (pool->refs[(size_t)ids[b]] <= 0) return PQKV_ERR_STATE;
  }
  // Blocks whose prefix is cached already (in that block or in another one)
  // are skipped; from the first prefix that is not cached on, every block is
  // a new entry and must not be cached under another key or repeated.
  PrefixKey k;
  k.parent = 0;
  int b0 = 0;
  for (; b0 < nfull; ++b0) {
    std::memcpy(k.tok, token_ids + (size_t)b0 * PQKV_BLOCK_SIZE, sizeof(k.tok));
    const auto it = pool->map.find(k);
    if (it == pool->map.end()) break;
    k.parent = pool->serial[(size_t)it->second];
  }
  for (int b = b0; b < nfull; ++b) {
    if (pool->cached[(size_t)ids[b]]) return PQKV_ERR_STATE;
    for (int c = b0; c < b; ++c)
      if (ids[c] == ids[b]) return PQKV_ERR_STATE;
  }
  try {
    pool->map.reserve(pool->map.size() + (size_t)(nfull - b0));
  } catch (...) {
    return PQKV_ERR_OOM;
  }
  for (int b = b0; b < nfull; ++b) {
    std::memcpy(k.tok, token_ids + (size_t)b * PQKV_BLOCK_SIZE, sizeof(k.tok));
    const int32_t id = ids[b];
    try {
      pool->map.emplace(k, id);
    } catch (...) {
      return PQKV_ERR_OOM;  // the entries made so far are complete and valid
    }
    pool->key[(size_t)id] = k;
    pool->serial[(size_t)id] = pool->next_serial++;
    pool->cached[(size_t)id] = 1;
    k.parent = pool->serial[(size_t)id];
  }
  return PQKV_OK;
}

int pqkv_pool_cow(pqkv_pool* pool, int32_t id, int32_t* new_id, int* copy_needed) {
  if (!pool || !new_id || !copy_needed || id < 0 || id >= pool->num_blocks) return PQKV_ERR_ARG;
  if (pool->refs[(size_t)id] <= 0) return PQKV_ERR_STATE;
  if (pool->refs[(size_t)id] == 1 && !pool->cached[(size_t)id]) {
    *new_id = id;
    *copy_needed = 0;
    return PQKV_OK;
  }
  if (pool->free_ids.empty() && pool->n_evictable == 0) return PQKV_ERR_OOM;
  const int32_t fresh = pool->take();
  if (--pool->refs[(size_t)id] == 0) pool->release(id);
  *new_id = fresh;
  *copy_needed = 1;
  return PQKV_OK;
}

int32_t pqkv_pool_refcount(const pqkv_pool* pool, int32_t id) {
  if (!pool || id < 0 || id >= pool->num_blocks) return -1;
  return pool->refs[(size_t)id];
}

int pqkv_build_slot_mapping(const int32_t* block_tables, int batch, int max_blocks_per_seq,
                            const int32_t* start_pos, const int32_t* num_new, int32_t* slots_out) {
  if (!block_tables || !start_pos || !num_new || !slots_out || batch < 0 || max_blocks_per_seq < 1)
    return PQKV_ERR_ARG;
  // validate first so that a rejected call writes nothing
  for (int b = 0; b < batch; ++b) {
    if (start_pos[b] < 0 || num_new[b] < 0) return PQKV_ERR_ARG;
    const int64_t last = (int64_t)start_pos[b] + num_new[b] - 1;
    if (num_new[b] > 0 && last / PQKV_BLOCK_SIZE >= max_blocks_per_seq) return PQKV_ERR_ARG;
    for (int64_t pos = start_pos[b]; pos <= last; pos += PQKV_BLOCK_SIZE) {
      if (block_tables[(size_t)b * max_blocks_per_seq + pos / PQKV_BLOCK_SIZE] < 0) return PQKV_ERR_ARG;
    }
    if (num_new[b] > 0 && block_tables[(size_t)b * max_blocks_per_seq + last / PQKV_BLOCK_SIZE] < 0)
      return PQKV_ERR_ARG;
  }
  size_t o = 0;
  for (int b = 0; b < batch; ++b) {
    const int32_t* row = block_tables + (size_t)b * max_blocks_per_seq;
    for (int i = 0; i < num_new[b]; ++i) {
      const int64_t pos = (int64_t)start_pos[b] + i;
      slots_out[o++] = row[pos / PQKV_BLOCK_SIZE] * PQKV_BLOCK_SIZE + (int32_t)(pos % PQKV_BLOCK_SIZE);
    }
  }
  return PQKV_OK;
}

}  // extern "C"
