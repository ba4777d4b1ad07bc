// blocks.cuh -- whole-block moves (copy-on-write copies, swap to / from host).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace pqkv {

// The four cache arrays and the bytes one block occupies in each.
struct BlockArrays {
  uint8_t* base[4];   // cache, scales, outliers_idx, outliers_val (unused: nullptr)
  uint64_t bytes[4];  // bytes of one block in each array (multiples of 16)
  uint64_t end[4];    // running sums of bytes[]: record offset where each region ends
  uint64_t rec;       // record bytes = end[3]
};

enum BlockMoveMode { kMoveCopy = 0, kMoveToHost = 1, kMoveFromHost = 2 };

// Fills `a` for a format; false if a needed array is missing or misaligned.
bool block_arrays(int kv_dtype, int H, int D, void* cache, void* scales, void* oidx, void* oval, BlockArrays& a);

// kMoveCopy: ids = pairs [n][2] (src, dst); otherwise ids [n] and host records [n][a.rec].
cudaError_t launch_block_move(int mode, const BlockArrays& a, const int32_t* ids, int n, int nb, void* host,
                              int32_t* err, int sms, cudaStream_t st);

}  // namespace pqkv
