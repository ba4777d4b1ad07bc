// prefill.cuh -- chunked-prefill attention over the paged cache (tcgen05).
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"

namespace pqkv {

struct PrefillParams {
  const void* q;                // [cu_q[B]][Hq][D]
  void* out;                    // same shape and type as q
  const uint8_t* cache;
  const uint8_t* scales;
  const uint8_t* oidx;
  const uint8_t* oval;
  const int32_t* cu_q;          // [B + 1] query-token offsets
  const int32_t* seq_lens;      // [B] cached positions, the chunk's own included
  const int32_t* block_tables;  // [B][maxblk]
  int32_t* err;
  int B, Hq, Hkv, G, nb, maxblk;
  int tiles_per_seq;            // 128-row query tiles per sequence (from the longest chunk)
  float scale_log2;             // softmax scale * log2(e)
  uint64_t timeout_ns;          // limit of a wait before the CTA gives up
  uint64_t drain_ns;            // after giving up: limit of the wait for work still in flight
};

cudaError_t launch_prefill(int kv_dtype, int D, bool q_bf16, const CUtensorMap& tmap16, const PrefillParams& p,
                           cudaStream_t st);
size_t prefill_smem_bytes(int kv_dtype, int D);

}  // namespace pqkv
