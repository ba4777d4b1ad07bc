// api.cu -- C ABI entry points: argument validation, TMA descriptors, launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>

#include "blocks.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "write.cuh"

namespace pqkv {
cudaError_t launch_decode(int kv_dtype, int D, bool q_bf16, int nt, const CUtensorMap& tmap, const DecodeParams& p,
                          int grid, cudaStream_t st);
size_t decode_smem_bytes(int kv_dtype, int D, int B, int nt);
size_t read_probe_smem_bytes(int B);
cudaError_t launch_read_probe(const uint8_t* cache, int kv_dtype, int nb, int H, int D, const int32_t* block_tables,
                              int maxblk, const int32_t* seq_lens, int B, uint32_t* checksum, int32_t* err,
                              uint64_t timeout_ns, int sms, cudaStream_t st);
}  // namespace pqkv

using namespace pqkv;

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded wait on one asynchronous copy

// Limit of the decode kernels' waits on their copies (pqkv_set_decode_wait_limit_ns).
std::atomic<uint64_t> g_decode_wait_ns{kWaitLimitNs};

bool is_kv_dtype(int t) { return t >= PQKV_DTYPE_FP16 && t <= PQKV_DTYPE_FP4_E2M1; }
bool is_16(int t) { return t == PQKV_DTYPE_FP16 || t == PQKV_DTYPE_BF16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  int sms = 0;
  int max_smem = 0;
};

bool device_info(DeviceInfo& out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev].sms == 0) {
    int sms = 0, smem = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    cache[dev].sms = sms;
    cache[dev].max_smem = smem;
  }
  out = cache[dev];
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// TMA descriptor over the cache viewed as rows of one token's K or V:
// [num_blocks * H * 2 * 16 rows][row bytes]; one box = 32 rows (K and V of one
// (block, head) pair) x up to 128 bytes, swizzled to the box row width.
bool make_cache_map(CUtensorMap* map, const void* cache, int kv_dtype, int nb, int H, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int row = row_bytes(kv_dtype, D);
  const int box_row = std::min(row, 128);
  const int esz = is_16(kv_dtype) ? 2 : 1;
  const CUtensorMapDataType dt = is_16(kv_dtype) ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const cuuint64_t dims[2] = {(cuuint64_t)(row / esz), (cuuint64_t)nb * H * 2 * 16};
  const cuuint64_t strides[1] = {(cuuint64_t)row};
  const cuuint32_t box[2] = {(cuuint32_t)(box_row / esz), 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_row == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : box_row == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
  const CUresult r = fn(map, dt, 2, const_cast<void*>(cache), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// TMA descriptor for the prefill's 16-bit operand tiles: the same rows, one box
// = 16 rows (the K or the V of one (block, head) pair) x 64 elements, 128-byte
// swizzle (the tensor cores' operand layout).
bool make_prefill_map(CUtensorMap* map, const void* cache, int kv_dtype, int nb, int H, int D) {
  auto fn = encode_fn();
  if (!fn || !is_16(kv_dtype)) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)nb * H * 2 * 16};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(cache), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Most recent descriptor per thread (the cache buffer rarely changes).
bool cached_cache_map(CUtensorMap* map, const void* cache, int kv_dtype, int nb, int H, int D) {
  struct Key {
    const void* p;
    int dt, nb, H, D, dev;
  };
  thread_local Key key{nullptr, -1, 0, 0, 0, -1};
  thread_local CUtensorMap last;
  int dev = 0;
  cudaGetDevice(&dev);
  if (key.p == cache && key.dt == kv_dtype && key.nb == nb && key.H == H && key.D == D && key.dev == dev) {
    *map = last;
    return true;
  }
  if (!make_cache_map(&last, cache, kv_dtype, nb, H, D)) return false;
  key = Key{cache, kv_dtype, nb, H, D, dev};
  *map = last;
  return true;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace = two partial-result slots per chunk of the split and one arrival
// word per chunk, all written by the decode kernel before it reads them (the
// words carry a per-launch tag); nothing in it needs to be initialized by the
// caller.

}  // namespace

namespace pqkv {
// The size and type checks of a decode call, shared by every decode entry point
// (the pointer and workspace checks follow in decode_impl).
int decode_check_sizes(int q_dtype, int batch, int q_len, int num_q_heads, int kv_dtype, int num_blocks,
                       int num_kv_heads, int head_dim, int max_blocks_per_seq, int split_blocks) {
  if (!is_kv_dtype(kv_dtype) || (q_dtype != PQKV_DTYPE_FP16 && q_dtype != PQKV_DTYPE_BF16)) return PQKV_ERR_ARG;
  if (is_16(kv_dtype) && q_dtype != kv_dtype) return PQKV_ERR_ARG;
  if (batch < 0 || batch > PQKV_MAX_BATCH || num_kv_heads < 1 || num_q_heads < 1 ||
      num_q_heads % num_kv_heads != 0 || q_len < 1 || q_len > 64 || num_q_heads / num_kv_heads > 8 ||
      (head_dim != 64 && head_dim != 128) ||
      num_blocks < 1 || max_blocks_per_seq < 1 || split_blocks < 0)
    return PQKV_ERR_ARG;
  return PQKV_OK;
}
}  // namespace pqkv

extern "C" {

int pqkv_version(void) { return 10000; }

void pqkv_set_decode_wait_limit_ns(uint64_t ns) { g_decode_wait_ns.store(ns ? ns : kWaitLimitNs); }

const char* pqkv_status_string(int status) {
  switch (status) {
    case PQKV_OK: return "ok";
    case PQKV_ERR_ARG: return "invalid argument";
    case PQKV_ERR_OOM: return "block pool exhausted";
    case PQKV_ERR_STATE: return "invalid block state";
    case PQKV_ERR_CUDA: return "CUDA error";
    case PQKV_ERR_SCRATCH: return "request exceeds the static scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

int pqkv_cache_layout(int kv_dtype, int num_blocks, int num_kv_heads, int head_dim, size_t out_bytes[4]) {
  if (!out_bytes || !is_kv_dtype(kv_dtype) || num_blocks < 1 || num_kv_heads < 1 ||
      (head_dim != 64 && head_dim != 128))
    return PQKV_ERR_ARG;
  const size_t pairs = (size_t)num_blocks * num_kv_heads;
  out_bytes[0] = pairs * 2 * PQKV_BLOCK_SIZE * (size_t)row_bytes(kv_dtype, head_dim);
  out_bytes[1] = out_bytes[2] = out_bytes[3] = 0;
  if (kv_dtype == PQKV_DTYPE_FP8_E4M3 || kv_dtype == PQKV_DTYPE_FP8_E5M2) out_bytes[1] = pairs * 4 * sizeof(float);
  if (kv_dtype == PQKV_DTYPE_FP4_E2M1) {
    out_bytes[1] = pairs * 2 * PQKV_BLOCK_SIZE * (size_t)(head_dim / PQKV_FP4_GROUP);
    out_bytes[2] = pairs * 2 * PQKV_FP4_IDX_STRIDE;
    out_bytes[3] = pairs * 2 * PQKV_BLOCK_SIZE * PQKV_FP4_OUTLIER_SLOTS * 2;
  }
  return PQKV_OK;
}

int pqkv_kv_cache_write(const void* k, const void* v, int in_dtype, int num_tokens, const int32_t* slot_mapping,
                        void* cache, void* scales, void* outliers_idx, void* outliers_val, int kv_dtype,
                        int num_blocks, int num_kv_heads, int head_dim, int32_t* err_flag, pqkv_stream_t stream) {
  if (!is_kv_dtype(kv_dtype) || (in_dtype != PQKV_DTYPE_FP16 && in_dtype != PQKV_DTYPE_BF16)) return PQKV_ERR_ARG;
  if (is_16(kv_dtype) && in_dtype != kv_dtype) return PQKV_ERR_ARG;
  if (num_tokens < 0 || num_blocks < 1 || num_kv_heads < 1 || (head_dim != 64 && head_dim != 128))
    return PQKV_ERR_ARG;
  if ((int64_t)num_blocks * PQKV_BLOCK_SIZE > INT32_MAX) return PQKV_ERR_ARG;
  if (num_tokens == 0) return PQKV_OK;
  if (!k || !v || !slot_mapping || !cache || !err_flag) return PQKV_ERR_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(cache)) return PQKV_ERR_ARG;
  if (!is_16(kv_dtype) && !scales) return PQKV_ERR_ARG;
  if (kv_dtype == PQKV_DTYPE_FP4_E2M1 && (!outliers_idx || !outliers_val)) return PQKV_ERR_ARG;
  WriteParams p;
  p.k = k;
  p.v = v;
  p.slots = slot_mapping;
  p.cache = static_cast<uint8_t*>(cache);
  p.scales = static_cast<uint8_t*>(scales);
  p.oidx = static_cast<uint8_t*>(outliers_idx);
  p.oval = static_cast<uint8_t*>(outliers_val);
  p.err = err_flag;
  p.T = num_tokens;
  p.nb = num_blocks;
  p.Hkv = num_kv_heads;
  const cudaError_t e = launch_write(kv_dtype, in_dtype, head_dim, p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PQKV_OK : PQKV_ERR_CUDA;
}

// Upper bound of the decode's units (each has two partial slots and one
// arrival word in the workspace): one per warp with the balanced split; with
// a fixed split, the split's chunks plus the warps' share boundaries inside them.
static size_t decode_chunks(int batch, int num_kv_heads, int max_blocks_per_seq, int split_blocks, int sms) {
  const size_t total_blocks = (size_t)batch * num_kv_heads * max_blocks_per_seq;
  const size_t warps = (size_t)sms * kDecodeWarps;
  return split_blocks > 0 ? (total_blocks + split_blocks - 1) / split_blocks + warps : warps;
}

// Launch tags of the decode's arrival words (40 bits): 0xFF, then a 31-bit
// launch counter that is never 0. An arrival word is (tag << 24) | pieces, so a
// word matches a tag only if its high 32 bits, read as a float, are at most
// -2^127 or a negative NaN (the top byte 0xFF), and not -inf (whose low bits
// would need the counter's bit 31). A zeroed word, or one left over from the
// partial outputs of a call with another layout (finite values, -inf row
// maxima), never matches; the counter repeats only after 2^31 - 1 launches.
static unsigned long long next_decode_epoch() {
  static std::atomic<unsigned long long> n{0};
  for (;;) {
    const unsigned long long c = (n.fetch_add(1) + 1) & 0x7FFFFFFFull;
    if (c != 0) return (0xFFull << 32) | c;
  }
}

size_t pqkv_decode_workspace_bytes(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                   int max_blocks_per_seq, int split_blocks) {
  if (batch < 1 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0 ||
      (head_dim != 64 && head_dim != 128) || max_blocks_per_seq < 1 || split_blocks < 0)
    return 0;
  const int G = num_q_heads / num_kv_heads;
  if (G > 16) return 0;  // columns of one pass: up to two tiles of 8
  DeviceInfo di;
  if (!device_info(di)) return 0;
  const size_t slot = round_up((size_t)G * head_dim + 2 * G, 4) * 4;
  const size_t chunks = decode_chunks(batch, num_kv_heads, max_blocks_per_seq, split_blocks, di.sms);
  return 2 * chunks * slot + chunks * sizeof(unsigned long long);  // partial slots, then arrival words
}

int pqkv_decode_workspace_init(void* workspace, size_t workspace_bytes, pqkv_stream_t stream) {
  if (!workspace && workspace_bytes) return PQKV_ERR_ARG;
  if (!workspace_bytes) return PQKV_OK;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PQKV_OK
             : PQKV_ERR_CUDA;
}

// Query tokens per decode pass: the G query heads of kp consecutive tokens fill
// up to 16 MMA columns (two tiles of 8 when more than 8 are used).
static int mq_tokens_per_pass(int q_len, int G) { return std::min(q_len, std::max(1, 16 / G)); }

size_t pqkv_multi_query_decode_workspace_bytes(int batch, int q_len, int num_q_heads, int num_kv_heads,
                                               int head_dim, int max_blocks_per_seq, int split_blocks) {
  if (q_len < 1 || q_len > 64 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0 ||
      num_q_heads / num_kv_heads > 8)
    return 0;
  const int kp = mq_tokens_per_pass(q_len, num_q_heads / num_kv_heads);
  return pqkv_decode_workspace_bytes(batch, num_q_heads * kp, num_kv_heads, head_dim, max_blocks_per_seq,
                                     split_blocks);
}


static int decode_impl(const void* q, int q_dtype, int batch, int q_len, int num_q_heads, const void* cache,
                       const void* scales, const void* outliers_idx, const void* outliers_val, int kv_dtype,
                       int num_blocks, int num_kv_heads, int head_dim, const int32_t* block_tables,
                       int max_blocks_per_seq, const int32_t* seq_lens, float scale, int split_blocks, void* out,
                       void* workspace, size_t workspace_bytes, int32_t* err_flag, pqkv_stream_t stream) {
  if (decode_check_sizes(q_dtype, batch, q_len, num_q_heads, kv_dtype, num_blocks, num_kv_heads, head_dim,
                         max_blocks_per_seq, split_blocks) != PQKV_OK)
    return PQKV_ERR_ARG;
  if (batch == 0) return PQKV_OK;
  if (!q || !cache || !block_tables || !seq_lens || !out || !workspace || !err_flag) return PQKV_ERR_ARG;
  if (!is_16(kv_dtype) && !scales) return PQKV_ERR_ARG;
  if (kv_dtype == PQKV_DTYPE_FP4_E2M1 && (!outliers_idx || !outliers_val)) return PQKV_ERR_ARG;
  if (!aligned16(cache) || (scales && !aligned16(scales)) || (outliers_idx && !aligned16(outliers_idx)) ||
      (outliers_val && !aligned16(outliers_val)) || !aligned16(q) || !aligned16(out))
    return PQKV_ERR_ARG;
  // flat block indices and TMA row coordinates must fit in int32
  if ((int64_t)batch * num_kv_heads * max_blocks_per_seq >= INT32_MAX ||
      (int64_t)num_blocks * num_kv_heads * 32 >= INT32_MAX)
    return PQKV_ERR_ARG;
  // A pass takes up to 16 MMA columns: the G query heads of kp consecutive
  // query tokens; more tokens take several passes, each reading the KV once.
  // The pieces hold one row per column of a pass.
  const int Gh = num_q_heads / num_kv_heads;
  const int kp = mq_tokens_per_pass(q_len, Gh);
  const size_t need = pqkv_decode_workspace_bytes(batch, num_q_heads * kp, num_kv_heads, head_dim,
                                                  max_blocks_per_seq, split_blocks);
  if (need == 0 || workspace_bytes < need) return PQKV_ERR_ARG;
  DeviceInfo di;
  if (!device_info(di)) return PQKV_ERR_CUDA;
  for (int nt = 1; nt <= (Gh * kp > 8 ? 2 : 1); ++nt)
    if (decode_smem_bytes(kv_dtype, head_dim, batch, nt) > (size_t)di.max_smem) return PQKV_ERR_ARG;
  CUtensorMap tmap;
  if (!cached_cache_map(&tmap, cache, kv_dtype, num_blocks, num_kv_heads, head_dim)) return PQKV_ERR_CUDA;
  DecodeParams p;
  p.q = q;
  p.out = out;
  p.scales = static_cast<const uint8_t*>(scales);
  p.oidx = static_cast<const uint8_t*>(outliers_idx);
  p.oval = static_cast<const uint8_t*>(outliers_val);
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.err = err_flag;
  p.partials = static_cast<float*>(workspace);
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.Gh = Gh;
  p.k = q_len;
  p.nb = num_blocks;
  p.maxblk = max_blocks_per_seq;
  p.split_blocks = split_blocks;
  p.slot_floats = (int)round_up((size_t)Gh * kp * head_dim + 2 * Gh * kp, 4);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_decode_wait_ns.load();
  p.drain_ns = kWaitLimitNs;
  // the arrival words follow the partial slots (16-byte aligned: slot_floats is a multiple of 4)
  const size_t chunks = decode_chunks(batch, num_kv_heads, max_blocks_per_seq, split_blocks, di.sms);
  p.counters = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) +
                                                     2 * chunks * (size_t)p.slot_floats * sizeof(float));
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // passes run in stream order; each kernel waits for the previous one before
  // touching the workspace (programmatic dependents wait for the full grid)
  for (int q0 = 0; q0 < q_len; q0 += kp) {
    p.q0 = q0;
    p.G = Gh * std::min(kp, q_len - q0);
    p.epoch = next_decode_epoch();
    const int nt = p.G > 8 ? 2 : 1;  // tiles of 8 columns
    const cudaError_t e = launch_decode(kv_dtype, head_dim, q_dtype == PQKV_DTYPE_BF16, nt, tmap, p, di.sms, st);
    if (e != cudaSuccess) return PQKV_ERR_CUDA;
  }
  return PQKV_OK;
}

int pqkv_paged_decode_attention(const void* q, int q_dtype, int batch, int num_q_heads, const void* cache,
                                const void* scales, const void* outliers_idx, const void* outliers_val,
                                int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                                const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
                                float scale, int split_blocks, void* out, void* workspace,
                                size_t workspace_bytes, int32_t* err_flag, pqkv_stream_t stream) {
  return decode_impl(q, q_dtype, batch, 1, num_q_heads, cache, scales, outliers_idx, outliers_val, kv_dtype,
                     num_blocks, num_kv_heads, head_dim, block_tables, max_blocks_per_seq, seq_lens, scale,
                     split_blocks, out, workspace, workspace_bytes, err_flag, stream);
}

int pqkv_paged_multi_query_decode_attention(const void* q, int q_dtype, int batch, int q_len, int num_q_heads,
                                            const void* cache, const void* scales, const void* outliers_idx,
                                            const void* outliers_val, int kv_dtype, int num_blocks,
                                            int num_kv_heads, int head_dim, const int32_t* block_tables,
                                            int max_blocks_per_seq, const int32_t* seq_lens, float scale,
                                            int split_blocks, void* out, void* workspace, size_t workspace_bytes,
                                            int32_t* err_flag, pqkv_stream_t stream) {
  return decode_impl(q, q_dtype, batch, q_len, num_q_heads, cache, scales, outliers_idx, outliers_val, kv_dtype,
                     num_blocks, num_kv_heads, head_dim, block_tables, max_blocks_per_seq, seq_lens, scale,
                     split_blocks, out, workspace, workspace_bytes, err_flag, stream);
}

size_t pqkv_block_record_bytes(int kv_dtype, int num_kv_heads, int head_dim) {
  if (!is_kv_dtype(kv_dtype) || num_kv_heads < 1 || (head_dim != 64 && head_dim != 128)) return 0;
  size_t b[4];
  if (pqkv_cache_layout(kv_dtype, 1, num_kv_heads, head_dim, b) != PQKV_OK) return 0;
  return b[0] + b[1] + b[2] + b[3];
}

static int block_move(int mode, void* cache, void* scales, void* outliers_idx, void* outliers_val, int kv_dtype,
                      int num_blocks, int num_kv_heads, int head_dim, const int32_t* ids, int num, void* host,
                      int32_t* err_flag, pqkv_stream_t stream) {
  if (!is_kv_dtype(kv_dtype) || num_blocks < 1 || num_kv_heads < 1 || (head_dim != 64 && head_dim != 128) ||
      num < 0)
    return PQKV_ERR_ARG;
  if (num == 0) return PQKV_OK;
  if (!ids || !err_flag || !cache) return PQKV_ERR_ARG;
  BlockArrays a;
  if (!block_arrays(kv_dtype, num_kv_heads, head_dim, cache, scales, outliers_idx, outliers_val, a))
    return PQKV_ERR_ARG;
  void* dev_host = nullptr;
  if (mode != kMoveCopy) {
    if (!host || !aligned16(host)) return PQKV_ERR_ARG;
    if (cudaHostGetDevicePointer(&dev_host, host, 0) != cudaSuccess || !aligned16(dev_host)) {
      (void)cudaGetLastError();  // clear the error this query left behind
      return PQKV_ERR_ARG;
    }
  }
  DeviceInfo di;
  if (!device_info(di)) return PQKV_ERR_CUDA;
  const cudaError_t e = launch_block_move(mode, a, ids, num, num_blocks, dev_host, err_flag, di.sms,
                                          reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PQKV_OK : PQKV_ERR_CUDA;
}

int pqkv_copy_blocks(void* cache, void* scales, void* outliers_idx, void* outliers_val, int kv_dtype,
                     int num_blocks, int num_kv_heads, int head_dim, const int32_t* pairs, int num_pairs,
                     int32_t* err_flag, pqkv_stream_t stream) {
  return block_move(kMoveCopy, cache, scales, outliers_idx, outliers_val, kv_dtype, num_blocks, num_kv_heads,
                    head_dim, pairs, num_pairs, nullptr, err_flag, stream);
}

int pqkv_swap_out(const void* cache, const void* scales, const void* outliers_idx, const void* outliers_val,
                  int kv_dtype, int num_blocks, int num_kv_heads, int head_dim, const int32_t* block_ids, int num,
                  void* host_records, int32_t* err_flag, pqkv_stream_t stream) {
  return block_move(kMoveToHost, const_cast<void*>(cache), const_cast<void*>(scales),
                    const_cast<void*>(outliers_idx), const_cast<void*>(outliers_val), kv_dtype, num_blocks,
                    num_kv_heads, head_dim, block_ids, num, host_records, err_flag, stream);
}

int pqkv_swap_in(void* cache, void* scales, void* outliers_idx, void* outliers_val, int kv_dtype, int num_blocks,
                 int num_kv_heads, int head_dim, const int32_t* block_ids, int num, const void* host_records,
                 int32_t* err_flag, pqkv_stream_t stream) {
  return block_move(kMoveFromHost, cache, scales, outliers_idx, outliers_val, kv_dtype, num_blocks, num_kv_heads,
                    head_dim, block_ids, num, const_cast<void*>(host_records), err_flag, stream);
}

int pqkv_paged_prefill_attention(const void* q, int q_dtype, int batch, int max_q_len, int num_q_heads,
                                 const int32_t* cu_q_lens, const void* cache, const void* scales,
                                 const void* outliers_idx, const void* outliers_val, int kv_dtype, int num_blocks,
                                 int num_kv_heads, int head_dim, const int32_t* block_tables,
                                 int max_blocks_per_seq, const int32_t* seq_lens, float scale, void* out,
                                 int32_t* err_flag, pqkv_stream_t stream) {
  if (!is_kv_dtype(kv_dtype) || (q_dtype != PQKV_DTYPE_FP16 && q_dtype != PQKV_DTYPE_BF16)) return PQKV_ERR_ARG;
  if (is_16(kv_dtype) && q_dtype != kv_dtype) return PQKV_ERR_ARG;
  if (batch < 0 || max_q_len < 1 || num_q_heads < 1 || num_kv_heads < 1 || num_blocks < 1 ||
      max_blocks_per_seq < 1 || (head_dim != 64 && head_dim != 128))
    return PQKV_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PQKV_ERR_ARG;
  const int G = num_q_heads / num_kv_heads;
  if (128 % G != 0) return PQKV_ERR_ARG;
  if (num_kv_heads > 65535 || !(scale == scale)) return PQKV_ERR_ARG;
  if (batch == 0) return PQKV_OK;
  const int64_t tiles = ((int64_t)max_q_len * G + 127) / 128;
  if (tiles * batch > INT32_MAX) return PQKV_ERR_ARG;
  if (!q || !cu_q_lens || !cache || !block_tables || !seq_lens || !out || !err_flag) return PQKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(cache)) return PQKV_ERR_ARG;
  if (!is_16(kv_dtype) && (!scales || !aligned16(scales))) return PQKV_ERR_ARG;
  if (kv_dtype == PQKV_DTYPE_FP4_E2M1 &&
      (!outliers_idx || !outliers_val || !aligned16(outliers_idx) || !aligned16(outliers_val)))
    return PQKV_ERR_ARG;
  DeviceInfo di;
  if (!device_info(di)) return PQKV_ERR_CUDA;
  if ((size_t)di.max_smem < prefill_smem_bytes(kv_dtype, head_dim)) return PQKV_ERR_CUDA;
  CUtensorMap tmap;
  std::memset(&tmap, 0, sizeof(tmap));
  if (is_16(kv_dtype) && !make_prefill_map(&tmap, cache, kv_dtype, num_blocks, num_kv_heads, head_dim))
    return PQKV_ERR_CUDA;
  PrefillParams p;
  p.q = q;
  p.out = out;
  p.cache = static_cast<const uint8_t*>(cache);
  p.scales = static_cast<const uint8_t*>(scales);
  p.oidx = static_cast<const uint8_t*>(outliers_idx);
  p.oval = static_cast<const uint8_t*>(outliers_val);
  p.cu_q = cu_q_lens;
  p.seq_lens = seq_lens;
  p.block_tables = block_tables;
  p.err = err_flag;
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = G;
  p.nb = num_blocks;
  p.maxblk = max_blocks_per_seq;
  p.tiles_per_seq = (int)tiles;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_decode_wait_ns.load();
  p.drain_ns = kWaitLimitNs;
  const cudaError_t e = launch_prefill(kv_dtype, head_dim, q_dtype == PQKV_DTYPE_BF16, tmap, p,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PQKV_OK : PQKV_ERR_CUDA;
}

int pqkv_read_probe(const void* cache, int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens, int batch,
                    uint32_t* checksum, int32_t* err_flag, pqkv_stream_t stream) {
  if (!is_kv_dtype(kv_dtype) || num_blocks < 1 || num_kv_heads < 1 || (head_dim != 64 && head_dim != 128) ||
      max_blocks_per_seq < 1 || batch < 0 || batch > PQKV_MAX_BATCH)
    return PQKV_ERR_ARG;
  if ((int64_t)batch * num_kv_heads * max_blocks_per_seq >= INT32_MAX) return PQKV_ERR_ARG;
  if (batch == 0) return PQKV_OK;
  if (!cache || !block_tables || !seq_lens || !checksum || !err_flag || !aligned16(cache)) return PQKV_ERR_ARG;
  DeviceInfo di;
  if (!device_info(di)) return PQKV_ERR_CUDA;
  if (read_probe_smem_bytes(batch) > (size_t)di.max_smem) return PQKV_ERR_ARG;
  const cudaError_t e = launch_read_probe(static_cast<const uint8_t*>(cache), kv_dtype, num_blocks, num_kv_heads,
                                          head_dim, block_tables, max_blocks_per_seq, seq_lens, batch, checksum,
                                          err_flag, kWaitLimitNs, di.sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PQKV_OK : PQKV_ERR_CUDA;
}

int pqkv_encode(const float* x, int64_t n, int code_dtype, uint8_t* codes, pqkv_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !codes))) return PQKV_ERR_ARG;
  if (code_dtype != PQKV_DTYPE_FP8_E4M3 && code_dtype != PQKV_DTYPE_FP8_E5M2 && code_dtype != PQKV_DTYPE_FP4_E2M1)
    return PQKV_ERR_ARG;
  const cudaError_t e = launch_encode(code_dtype, x, n, codes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PQKV_OK : PQKV_ERR_CUDA;
}

}  // extern "C"
