// write.cuh -- parameters and launchers of the cache-write and encode kernels.
#pragma once

#include "common.cuh"

namespace pqkv {

struct WriteParams {
  const void* k;
  const void* v;
  const int32_t* slots;
  uint8_t* cache;
  uint8_t* scales;
  uint8_t* oidx;
  uint8_t* oval;
  int32_t* err;
  int T, nb, Hkv;
  int tpw;  // tokens per warp window (set by the launcher)
};

cudaError_t launch_write(int kv_dtype, int in_dtype, int D, const WriteParams& p, cudaStream_t st);
cudaError_t launch_encode(int code_dtype, const float* x, int64_t n, uint8_t* out, cudaStream_t st);

}  // namespace pqkv
