// noalloc.cu -- paged decode attention for callers that cannot allocate
// device memory.
//
// Some callers cannot hand the library a workspace: code that runs inside a
// host whose device memory is fully reserved by its own pool, or a
// latency-critical path where a cudaMalloc (which may synchronize the device)
// is not acceptable. For them the decode's scratch (the split plan and the
// partial softmax results) lives in one file-scope device array of fixed size,
// PQKV_NOALLOC_SCRATCH_BYTES, that every GPU loading this library holds until
// the process exits. Nothing here allocates: no cudaMalloc / cudaFree and no
// allocating library routine.
//
// In host code the array's name is only a host-side stand-in; its device
// address comes from cudaGetSymbolAddress, taken once per device with that
// device current (on the first call made on the device).
#include <mutex>

#include "../../include/pqkv.h"
#include <cuda_runtime.h>

static __device__ __align__(256) unsigned char g_pqkv_noalloc_scratch[PQKV_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device (null on error).
void* scratch_address() {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pqkv_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" int pqkv_paged_decode_attention_noalloc(const void* q, int q_dtype, int batch, int num_q_heads,
                                                   const void* cache, const void* scales,
                                                   const void* outliers_idx, const void* outliers_val,
                                                   int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                                                   const int32_t* block_tables, int max_blocks_per_seq,
                                                   const int32_t* seq_lens, float scale, int split_blocks,
                                                   void* out, int32_t* err_flag, pqkv_stream_t stream) {
  if (batch == 0) return PQKV_OK;
  const size_t need = pqkv_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                                                  split_blocks);
  if (need == 0) return PQKV_ERR_ARG;
  if (need > (size_t)PQKV_NOALLOC_SCRATCH_BYTES) return PQKV_ERR_SCRATCH;
  void* ws = scratch_address();
  if (!ws) return PQKV_ERR_CUDA;
  // The decode writes every scratch byte it later reads (plan first, then the
  // partial slots), so no part of the array has to start at zero.
  return pqkv_paged_decode_attention(q, q_dtype, batch, num_q_heads, cache, scales, outliers_idx, outliers_val,
                                     kv_dtype, num_blocks, num_kv_heads, head_dim, block_tables,
                                     max_blocks_per_seq, seq_lens, scale, split_blocks, out, ws,
                                     (size_t)PQKV_NOALLOC_SCRATCH_BYTES, err_flag, stream);
}
