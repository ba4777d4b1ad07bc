// blocks.cu -- whole-block moves: copy-on-write copies inside the cache and
// swaps between the cache and page-locked host memory.
//
// "vLLM" glossary: "PagedAttention" (blocks shared across sequences for beam
// search and parallel sampling: a sequence that writes into a shared block
// first takes its own copy), "Preemption support" (KV cache blocks swapped out
// to CPU RAM and back), "CPU offloading".
//
// A block is the same region of each of the four cache arrays (codes, scales,
// outlier indices, outlier values), each region contiguous and a multiple of
// 16 bytes; a block's "record" is the concatenation of its regions. One CTA
// moves one record at a time (grid-stride over records), its threads striding
// over the record's 16-byte chunks so that neighbouring threads touch
// neighbouring bytes, each thread keeping several chunks in flight (HBM, or
// host memory over the host link).
#include "blocks.cuh"
#include "common.cuh"

namespace pqkv {

namespace {

constexpr int kMoveThreads = 256;
constexpr int kMoveUnroll = 8;

struct MoveParams {
  BlockArrays a;
  const int32_t* ids;  // kMoveCopy: pairs [n][2] (src, dst); otherwise [n]
  uint8_t* host;       // records [n][rec] (device-accessible host pointer)
  int32_t* err;
  int n, nb;
};

// Address of byte `off` (16-aligned) of block `id`'s record in the cache arrays.
__device__ __forceinline__ uint8_t* rec_addr(const BlockArrays& a, int id, uint64_t off) {
  int s = 0;
  uint64_t lo = 0;
  if (off >= a.end[0]) { s = 1; lo = a.end[0]; }
  if (off >= a.end[1]) { s = 2; lo = a.end[1]; }
  if (off >= a.end[2]) { s = 3; lo = a.end[2]; }
  return a.base[s] + (uint64_t)id * a.bytes[s] + (off - lo);
}

template <int MODE>
__global__ void __launch_bounds__(kMoveThreads) block_move_kernel(const MoveParams p) {
  const uint32_t cpr = (uint32_t)(p.a.rec / 16);  // chunks per record
  for (int r = blockIdx.x; r < p.n; r += gridDim.x) {
    int src_id, dst_id;
    if constexpr (MODE == kMoveCopy) {
      src_id = p.ids[2 * r];
      dst_id = p.ids[2 * r + 1];
    } else {
      src_id = dst_id = p.ids[r];
    }
    if (src_id < 0 || src_id >= p.nb || dst_id < 0 || dst_id >= p.nb) {
      if (threadIdx.x == 0) raise_flag(p.err, PQKV_DEVERR_BLOCK_ID);
      continue;
    }
    uint8_t* hrec = (MODE == kMoveCopy) ? nullptr : p.host + (uint64_t)r * p.a.rec;
    for (uint32_t c0 = threadIdx.x; c0 < cpr; c0 += kMoveThreads * kMoveUnroll) {
      uint4 v[kMoveUnroll];
#pragma unroll
      for (int u = 0; u < kMoveUnroll; ++u) {
        const uint32_t c = c0 + u * kMoveThreads;
        if (c >= cpr) break;
        const uint64_t off = (uint64_t)c * 16;
        const uint8_t* src = (MODE == kMoveFromHost) ? hrec + off : rec_addr(p.a, src_id, off);
        v[u] = __ldcs(reinterpret_cast<const uint4*>(src));
      }
#pragma unroll
      for (int u = 0; u < kMoveUnroll; ++u) {
        const uint32_t c = c0 + u * kMoveThreads;
        if (c >= cpr) break;
        const uint64_t off = (uint64_t)c * 16;
        uint8_t* dst = (MODE == kMoveToHost) ? hrec + off : rec_addr(p.a, dst_id, off);
        __stcs(reinterpret_cast<uint4*>(dst), v[u]);
      }
    }
  }
}

}  // namespace

// Per-block bytes of each cache array (same sizes as the cache layout for one block).
bool block_arrays(int kv_dtype, int H, int D, void* cache, void* scales, void* oidx, void* oval, BlockArrays& a) {
  const uint64_t pairs = (uint64_t)H;
  a.bytes[0] = pairs * 2 * kBlock * (uint64_t)row_bytes(kv_dtype, D);
  a.bytes[1] = a.bytes[2] = a.bytes[3] = 0;
  if (kv_dtype == PQKV_DTYPE_FP8_E4M3 || kv_dtype == PQKV_DTYPE_FP8_E5M2) a.bytes[1] = pairs * 16;
  if (kv_dtype == PQKV_DTYPE_FP4_E2M1) {
    a.bytes[1] = pairs * 2 * kBlock * (uint64_t)(D / PQKV_FP4_GROUP);
    a.bytes[2] = pairs * 2 * PQKV_FP4_IDX_STRIDE;
    a.bytes[3] = pairs * 2 * kBlock * PQKV_FP4_OUTLIER_SLOTS * 2;
  }
  void* ptr[4] = {cache, scales, oidx, oval};
  uint64_t run = 0;
  for (int s = 0; s < 4; ++s) {
    if (a.bytes[s] != 0 && !ptr[s]) return false;
    if ((a.bytes[s] & 15u) != 0) return false;
    if (a.bytes[s] != 0 && (reinterpret_cast<uintptr_t>(ptr[s]) & 15u) != 0) return false;
    a.base[s] = static_cast<uint8_t*>(ptr[s]);
    run += a.bytes[s];
    a.end[s] = run;
  }
  a.rec = run;
  return true;
}

cudaError_t launch_block_move(int mode, const BlockArrays& a, const int32_t* ids, int n, int nb, void* host,
                              int32_t* err, int sms, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  MoveParams p;
  p.a = a;
  p.ids = ids;
  p.host = static_cast<uint8_t*>(host);
  p.err = err;
  p.n = n;
  p.nb = nb;
  const int grid = n < sms * 8 ? n : sms * 8;
  switch (mode) {
    case kMoveCopy: block_move_kernel<kMoveCopy><<<grid, kMoveThreads, 0, st>>>(p); break;
    case kMoveToHost: block_move_kernel<kMoveToHost><<<grid, kMoveThreads, 0, st>>>(p); break;
    default: block_move_kernel<kMoveFromHost><<<grid, kMoveThreads, 0, st>>>(p); break;
  }
  return cudaGetLastError();
}

}  // namespace pqkv
