// noalloc.cu -- paged decode attention for callers that cannot allocate
// device memory.
//
// Some callers cannot hand the library a workspace: code that runs inside a
// host whose device memory is fully reserved by its own pool, or a
// latency-critical path where a cudaMalloc (which may synchronize the device)
// is not acceptable. For them the decode's scratch (the partial softmax results
// of split pairs and the pairs' arrival words) lives in one file-scope device
// array of fixed size, PQKV_NOALLOC_SCRATCH_BYTES, that every GPU loading this
// library holds until the process exits. Nothing here allocates: no cudaMalloc
// / cudaFree and no allocating library routine.
//
// In host code the array's name is only a host-side stand-in; its device
// address comes from cudaGetSymbolAddress, taken once per device with that
// device current (on the first call made on the device).
#include <cstring>
#include <mutex>

#include "../../include/pqkv.h"
#include <cuda_runtime.h>

static __device__ __align__(256) unsigned char g_pqkv_noalloc_scratch[PQKV_NOALLOC_SCRATCH_BYTES];

namespace pqkv {
int decode_check_sizes(int q_dtype, int batch, int q_len, int num_q_heads, int kv_dtype, int num_blocks,
                       int num_kv_heads, int head_dim, int max_blocks_per_seq, int split_blocks);
}  // namespace pqkv

namespace {

constexpr int kMaxDevices = 64;

// The sizes that fix where in the scratch a call keeps its partial results and
// its arrival words.
struct Layout {
  int batch, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, split_blocks;
  bool operator==(const Layout& o) const { return std::memcmp(this, &o, sizeof(Layout)) == 0; }
};

struct DeviceScratch {
  void* addr = nullptr;  // device address of the array on this device
  bool have_layout = false;
  Layout last{};         // layout of the previous call on this device
};

std::mutex g_mu;
DeviceScratch g_dev[kMaxDevices];

}  // namespace

extern "C" int pqkv_paged_decode_attention_noalloc(const void* q, int q_dtype, int batch, int num_q_heads,
                                                   const void* cache, const void* scales,
                                                   const void* outliers_idx, const void* outliers_val,
                                                   int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                                                   const int32_t* block_tables, int max_blocks_per_seq,
                                                   const int32_t* seq_lens, float scale, int split_blocks,
                                                   void* out, int32_t* err_flag, pqkv_stream_t stream) {
  // the same size checks as pqkv_paged_decode_attention, before the scratch limit
  if (pqkv::decode_check_sizes(q_dtype, batch, 1, num_q_heads, kv_dtype, num_blocks, num_kv_heads, head_dim,
                               max_blocks_per_seq, split_blocks) != PQKV_OK)
    return PQKV_ERR_ARG;
  if (batch == 0) return PQKV_OK;
  const size_t need = pqkv_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                                                  split_blocks);
  if (need == 0) return PQKV_ERR_ARG;
  if (need > (size_t)PQKV_NOALLOC_SCRATCH_BYTES) return PQKV_ERR_SCRATCH;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PQKV_ERR_CUDA;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceScratch& d = g_dev[dev];
    if (!d.addr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_pqkv_noalloc_scratch) != cudaSuccess) return PQKV_ERR_CUDA;
      d.addr = p;
    }
    ws = d.addr;
    // A split pair counts its pieces in an arrival word tagged with the
    // launch; words written by an earlier launch never match the tag. Where
    // those words sit depends on the layout, so after a call with another
    // layout the words of this one may hold that call's partial results, which
    // could match a tag by chance. Clearing the region this call uses (a
    // device memset, no allocation) whenever the layout changes leaves only
    // zeros or this layout's own earlier words there, and neither matches.
    const Layout cur{batch, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, split_blocks};
    if (!d.have_layout || !(d.last == cur)) {
      if (cudaMemsetAsync(ws, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PQKV_ERR_CUDA;
      d.last = cur;
      d.have_layout = true;
    }
  }
  return pqkv_paged_decode_attention(q, q_dtype, batch, num_q_heads, cache, scales, outliers_idx, outliers_val,
                                     kv_dtype, num_blocks, num_kv_heads, head_dim, block_tables,
                                     max_blocks_per_seq, seq_lens, scale, split_blocks, out, ws,
                                     (size_t)PQKV_NOALLOC_SCRATCH_BYTES, err_flag, stream);
}
