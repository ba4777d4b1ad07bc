// pool.cpp -- host block-pool allocator and slot-mapping helper.
//
// "vLLM" glossary, "PagedAttention": the KV cache is held in fixed-size blocks
// mapped from logical to physical ids and shared across sequences;
// "Continuous batching": finished sequences return their blocks to the pool.
// "vLLM v0.7.2" field report, "Field Observations": block pool exhaustion.
// Every operation is O(1) per block id and all-or-nothing.
#include <climits>
#include <cstdint>
#include <new>
#include <vector>

#include "../../include/pqkv.h"

struct pqkv_pool {
  int32_t num_blocks;
  std::vector<int32_t> free_ids;  // stack; back() is handed out next
  std::vector<int32_t> refs;
};

extern "C" {

int pqkv_pool_create(int32_t num_blocks, pqkv_pool** out_pool) {
  if (!out_pool || num_blocks < 1) return PQKV_ERR_ARG;
  pqkv_pool* p = new (std::nothrow) pqkv_pool;
  if (!p) return PQKV_ERR_OOM;
  try {
    p->num_blocks = num_blocks;
    p->refs.assign((size_t)num_blocks, 0);
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
  if ((size_t)n > pool->free_ids.size()) return PQKV_ERR_OOM;
  for (int i = 0; i < n; ++i) {
    const int32_t id = pool->free_ids.back();
    pool->free_ids.pop_back();
    pool->refs[(size_t)id] = 1;
    ids_out[i] = id;
  }
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
      pool->free_ids.push_back(ids[i]);
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
