// write.cu -- quantizing paged cache write for sm_100a.
//
// Method: "vLLM 0.7 Ships Unified KV Cache Compression", "Technical Breakdown:
// Dynamic Quantization with Outlier Retention", steps 1-3 (FP4 with outlier
// channels in an FP16 buffer); "vLLM v0.7.2" field report, "Deconstructing the
// v0.7.2 Architecture" (FP8 E4M3/E5M2 KV cache, 16-token blocks); "vLLM"
// glossary, "PagedAttention" (slot -> physical block). Readings of the pages
// (statistics, scale granularity, append rule) are stated in include/pqkv.h.
//
// Quantized formats work on runs: maximal chains of consecutive tokens whose
// slots increase by one inside one block. A warp owns a window of 32 tokens of
// one KV head and processes, one after the other, the runs that start in it.
// All rounding follows the stated fp32 steps: IEEE division (__fdiv_rn),
// hardware cvt with round-to-nearest-even and saturation; the FP4 outlier
// statistics are summed in fp64 in channel order on one lane.
#include <algorithm>

#include "write.cuh"

namespace pqkv {


namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

template <bool INBF16>
__device__ __forceinline__ float in_at(const void* x, size_t i) {
  if constexpr (INBF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(x)[i]);
  else
    return __half2float(reinterpret_cast<const __half*>(x)[i]);
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  return lo_half(dec_fp8x2<PQKV_DTYPE_FP8_E4M3>(code & 0xFFu));
}

template <int KVF>
__device__ __forceinline__ float fp8_value(uint32_t code) {
  return lo_half(dec_fp8x2<KVF>(code & 0xFFu));
}

// Run discovery for the window of 32 tokens owned by this warp. Returns the
// ballot of lanes whose token starts a run; raises SLOT / RUN error bits.
__device__ __forceinline__ uint32_t run_starts(const WriteParams& p, int t, bool mine, bool report) {
  const int lim = p.nb * kBlock;
  const int s = (mine && t < p.T) ? p.slots[t] : -1;
  const bool valid = (s >= 0 && s < lim);
  if (report && s >= lim) raise_flag(p.err, PQKV_DEVERR_SLOT);
  const int ps = (mine && t > 0 && t - 1 < p.T) ? p.slots[t - 1] : -1;
  const bool pvalid = (ps >= 0 && ps < lim);
  const bool cont = valid && pvalid && s == ps + 1 && (s & (kBlock - 1)) != 0;
  const bool start = valid && !cont;
  if (report && start && pvalid && (ps >> 4) == (s >> 4)) raise_flag(p.err, PQKV_DEVERR_RUN);
  return __ballot_sync(kFull, start);
}

// Length of the run starting at token ts with slot s0 (all lanes get it).
__device__ __forceinline__ int run_length(const WriteParams& p, int ts, int s0, int lane) {
  const int room = kBlock - (s0 & (kBlock - 1));
  bool ok = false;
  if (lane < room) {
    const int t = ts + lane;
    ok = (t < p.T) && p.slots[t] == s0 + lane;
  }
  const uint32_t m = __ballot_sync(kFull, ok);
  return __ffs(~m) - 1;  // bit 0 is always set
}

}  // namespace

// ---- 16-bit formats: one warp copies the K and V rows of one (token, head) ----
template <int D>
__global__ void __launch_bounds__(256) write16_kernel(const WriteParams p) {
  // inputs may come from the previous kernel; let the next one start launching
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long wid = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= (long)p.T * p.Hkv) return;
  const int t = (int)(wid / p.Hkv), h = (int)(wid % p.Hkv);
  const int s = p.slots[t];
  if (s < 0) return;
  if (s >= p.nb * kBlock) {
    if (h == 0 && lane == 0) raise_flag(p.err, PQKV_DEVERR_SLOT);
    return;
  }
  constexpr int kChunks = 2 * D / 16;  // 16-byte pieces per row
  if (lane >= 2 * kChunks) return;
  const int kv = lane / kChunks, c = lane % kChunks;
  const uint4* src = reinterpret_cast<const uint4*>(kv ? p.v : p.k) + ((size_t)t * p.Hkv + h) * kChunks + c;
  const size_t row = ((((size_t)(s >> 4) * p.Hkv + h) * 2 + kv) * kBlock + (s & 15));
  uint4* dst = reinterpret_cast<uint4*>(p.cache) + row * kChunks + c;
  *dst = __ldg(src);
}

// ---- FP8: absmax scale per (block, head, K|V), grown on append ----
template <int KVF, int D, bool INBF16>
__global__ void __launch_bounds__(128) write_fp8_kernel(const WriteParams p) {
  // inputs may come from the previous kernel; let the next one start launching
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int CPL = D / 32;  // channels per lane
  constexpr float kMax = (KVF == PQKV_DTYPE_FP8_E4M3) ? 448.0f : 57344.0f;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int win = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, kv = blockIdx.z;
  const int t = win * p.tpw + lane;
  uint32_t starts = run_starts(p, t, lane < p.tpw, h == 0 && kv == 0);
  while (starts) {
    const int i = __ffs(starts) - 1;
    starts &= starts - 1;
    const int ts = win * p.tpw + i;
    const int s0 = p.slots[ts];
    const int n = run_length(p, ts, s0, lane);
    const int blk = s0 >> 4, off0 = s0 & 15;
    const size_t pair = (size_t)blk * p.Hkv + h;
    {
      const void* x = kv ? p.v : p.k;
      float xs[kBlock][CPL];
      float a = 0.f;
#pragma unroll
      for (int j = 0; j < kBlock; ++j) {
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
          xs[j][e] = (j < n) ? in_at<INBF16>(x, ((size_t)(ts + j) * p.Hkv + h) * D + lane * CPL + e) : 0.f;
          a = fmaxf(a, fabsf(xs[j][e]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
      const float s_run = __fdiv_rn(a, kMax);
      float* sp = reinterpret_cast<float*>(p.scales) + pair * 4 + kv;
      uint8_t* tile = p.cache + (pair * 2 + kv) * kBlock * D;
      float s = s_run;
      if (off0 > 0) {
        const float s_old = *sp;
        s = fmaxf(s_old, s_run);
        if (s > s_old) {
          for (int r = 0; r < off0; ++r) {
            uint8_t* row = tile + r * D + lane * CPL;
            float y[CPL];
#pragma unroll
            for (int e = 0; e < CPL; ++e) y[e] = __fdiv_rn(__fmul_rn(fp8_value<KVF>(row[e]), s_old), s);
            if constexpr (CPL == 4) {
              const uint32_t c = enc_fp8x2<KVF>(y[0], y[1]) | (enc_fp8x2<KVF>(y[2], y[3]) << 16);
              *reinterpret_cast<uint32_t*>(row) = c;
            } else {
              *reinterpret_cast<uint16_t*>(row) = (uint16_t)enc_fp8x2<KVF>(y[0], y[1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) *sp = s;
#pragma unroll
      for (int j = 0; j < kBlock; ++j) {
        if (j >= n) break;
        uint8_t* row = tile + (off0 + j) * D + lane * CPL;
        float y[CPL];
#pragma unroll
        for (int e = 0; e < CPL; ++e) y[e] = (s > 0.f) ? __fdiv_rn(xs[j][e], s) : 0.f;
        uint32_t c;
        if constexpr (CPL == 4) {
          c = enc_fp8x2<KVF>(y[0], y[1]) | (enc_fp8x2<KVF>(y[2], y[3]) << 16);
          if (!(s > 0.f)) c = 0;
          *reinterpret_cast<uint32_t*>(row) = c;
        } else {
          c = enc_fp8x2<KVF>(y[0], y[1]);
          if (!(s > 0.f)) c = 0;
          *reinterpret_cast<uint16_t*>(row) = (uint16_t)c;
        }
      }
    }
  }
}

// ---- FP4 E2M1 + FP16 outlier channels ----
template <int D, bool INBF16>
__global__ void __launch_bounds__(128) write_fp4_kernel(const WriteParams p) {
  // inputs may come from the previous kernel; let the next one start launching
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int CPL = D / 32;          // channels per lane
  constexpr int LPG = kGroup / CPL;    // lanes per 16-channel group
  __shared__ float s_norm[4][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int win = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, kv = blockIdx.z;
  const int t = win * p.tpw + lane;
  uint32_t starts = run_starts(p, t, lane < p.tpw, h == 0 && kv == 0);
  while (starts) {
    const int i = __ffs(starts) - 1;
    starts &= starts - 1;
    const int ts = win * p.tpw + i;
    const int s0 = p.slots[ts];
    const int n = run_length(p, ts, s0, lane);
    const int blk = s0 >> 4, off0 = s0 & 15;
    const size_t pair = (size_t)blk * p.Hkv + h;
    {
      const void* x = kv ? p.v : p.k;
      const size_t tile = pair * 2 + kv;  // (block, head, K|V) index
      float xs[kBlock][CPL];
      float nrm[CPL];
#pragma unroll
      for (int e = 0; e < CPL; ++e) nrm[e] = 0.f;
#pragma unroll
      for (int j = 0; j < kBlock; ++j) {
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
          xs[j][e] = (j < n) ? in_at<INBF16>(x, ((size_t)(ts + j) * p.Hkv + h) * D + lane * CPL + e) : 0.f;
          nrm[e] = fmaxf(nrm[e], fabsf(xs[j][e]));
        }
      }
      uint8_t* idxp = p.oidx + tile * kIdxStride;
      int oc[kOutSlots];  // outlier channels (>= D: empty)
      if (off0 == 0) {
        // step 1: channel norms; step 2: mu + 3.2 sigma over the D norms (fp64, channel order)
#pragma unroll
        for (int e = 0; e < CPL; ++e) s_norm[warp][lane * CPL + e] = nrm[e];
        __syncwarp();
        double acc = 0.0;
        if (lane == 0) {
          for (int c = 0; c < D; ++c) acc = __dadd_rn(acc, (double)s_norm[warp][c]);
        } else if (lane == 1) {
          for (int c = 0; c < D; ++c) {
            const double v = (double)s_norm[warp][c];
            acc = __dadd_rn(acc, __dmul_rn(v, v));
          }
        }
        const double s2 = __shfl_sync(kFull, acc, 1);
        double thr = 0.0;
        if (lane == 0) {
          const double mu = __ddiv_rn(acc, (double)D);
          double var = __dsub_rn(__ddiv_rn(s2, (double)D), __dmul_rn(mu, mu));
          if (var < 0.0) var = 0.0;
          thr = __dadd_rn(mu, __dmul_rn(3.2, __dsqrt_rn(var)));
        }
        thr = __shfl_sync(kFull, thr, 0);
        __syncwarp();
        // keep at most 4: largest norm first, ties to the lower channel
        uint32_t cand = 0;
#pragma unroll
        for (int e = 0; e < CPL; ++e)
          if ((double)nrm[e] >= thr) cand |= 1u << e;
        int nsel = 0;
#pragma unroll
        for (int r = 0; r < kOutSlots; ++r) oc[r] = 0xFF;
        for (int r = 0; r < kOutSlots; ++r) {
          float bv = -1.f;
          int bc = 0x7FFFFFFF;
#pragma unroll
          for (int e = 0; e < CPL; ++e)
            if ((cand >> e) & 1u) {
              if (nrm[e] > bv) { bv = nrm[e]; bc = lane * CPL + e; }
            }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int occ = __shfl_xor_sync(kFull, bc, o);
            if (ov > bv || (ov == bv && occ < bc)) { bv = ov; bc = occ; }
          }
          if (bc == 0x7FFFFFFF) break;
          oc[nsel++] = bc;
          if (bc / CPL == lane) cand &= ~(1u << (bc % CPL));
        }
        // ascending order
#pragma unroll
        for (int a2 = 1; a2 < kOutSlots; ++a2)
#pragma unroll
          for (int b2 = kOutSlots - 1; b2 >= a2; --b2)
            if (oc[b2 - 1] > oc[b2]) { const int tmp = oc[b2]; oc[b2] = oc[b2 - 1]; oc[b2 - 1] = tmp; }
        if (lane == 0) {
          const uint32_t lo = (uint32_t)oc[0] | ((uint32_t)oc[1] << 8) | ((uint32_t)oc[2] << 16) | ((uint32_t)oc[3] << 24);
          reinterpret_cast<uint32_t*>(idxp)[0] = lo;
          reinterpret_cast<uint32_t*>(idxp)[1] = 0xFFFFFFFFu;
        }
      } else {
        const uint32_t lo = *reinterpret_cast<const uint32_t*>(idxp);
#pragma unroll
        for (int r = 0; r < kOutSlots; ++r) oc[r] = (lo >> (8 * r)) & 0xFF;
      }
      bool is_out[CPL];
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        const int c = lane * CPL + e;
        is_out[e] = (c == oc[0]) || (c == oc[1]) || (c == oc[2]) || (c == oc[3]);
      }
      // step 3: per token, fp16 outlier values, E4M3 group scales, E2M1 codes
      uint32_t vpend = 0;  // V codes of the even token of a pair, stored with its partner
#pragma unroll
      for (int j = 0; j < kBlock; ++j) {
        if (j >= n) break;
        const int row = off0 + j;
        // outlier buffer: lane r (< 4) stores slot r of this token
        {
          float ov = 0.f;
          int owner = 0, el = 0;
          const int r = lane & 3;
          const int c = oc[r];
          if (c < D) { owner = c / CPL; el = c % CPL; }
          float mine[CPL];
#pragma unroll
          for (int e = 0; e < CPL; ++e) mine[e] = xs[j][e];
          float got = 0.f;
#pragma unroll
          for (int e = 0; e < CPL; ++e) {
            const float v = __shfl_sync(kFull, mine[e], owner);
            if (e == el) got = v;
          }
          ov = (c < D) ? got : 0.f;
          if (lane < kOutSlots) {
            __half hv = (c < D) ? __float2half_rn(ov) : __ushort_as_half((unsigned short)0);
            reinterpret_cast<__half*>(p.oval)[(tile * kBlock + row) * kOutSlots + lane] = hv;
          }
        }
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < CPL; ++e)
          if (!is_out[e]) a = fmaxf(a, fabsf(xs[j][e]));
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
        const uint32_t sc = enc_fp8x2<PQKV_DTYPE_FP8_E4M3>(__fdiv_rn(a, 6.0f), 0.f) & 0xFFu;
        const float sd = e4m3_value(sc);
        float y[CPL];
#pragma unroll
        for (int e = 0; e < CPL; ++e) y[e] = (is_out[e] || sd == 0.f) ? 0.f : __fdiv_rn(xs[j][e], sd);
        const uint32_t c01 = enc_e2m1x2(y[0], y[1]);
        const uint32_t c23 = (CPL == 4) ? enc_e2m1x2(y[2], y[3]) : 0u;
        if (kv == 0) {
          // K: one row per token, channel 2i in the low nibble of byte i
          uint8_t* crow = p.cache + (tile * kBlock + row) * (D / 2) + lane * (CPL / 2);
          if constexpr (CPL == 4)
            *reinterpret_cast<uint16_t*>(crow) = (uint16_t)(c01 | (c23 << 8));
          else
            *crow = (uint8_t)c01;
        } else {
          // V: a byte holds one channel of a token pair (even token in the low
          // nibble). Pairs inside the run are stored whole; a pair split by the
          // run's ends keeps the other token's nibbles.
          const uint32_t cw = (c01 & 0xFu) | ((c01 >> 4) << 8) | ((c23 & 0xFu) << 16) | ((c23 >> 4) << 24);
          const int pr = (row < 8) ? (row & ~1) : (((row - 8) & ~1) + 1);
          const int cb = lane * CPL;
          uint8_t* vb = p.cache + (tile * kBlock + 8 * (cb / (D / 2)) + pr) * (D / 2) + cb % (D / 2);
          const bool odd = row & 1;
          if (!odd && j + 1 < n) {
            vpend = cw;
          } else {
            const int sh = odd ? 4 : 0;
            uint32_t keep = odd ? 0x0F0F0F0Fu : 0xF0F0F0F0u, put = cw << sh;
            if (odd && j > 0) { keep = 0u; put |= vpend; }
            if constexpr (CPL == 4) {
              uint32_t* w = reinterpret_cast<uint32_t*>(vb);
              *w = (keep ? (*w & keep) : 0u) | put;
            } else {
              uint16_t* w = reinterpret_cast<uint16_t*>(vb);
              *w = (uint16_t)((keep ? (*w & keep) : 0u) | put);
            }
          }
        }
        if ((lane % LPG) == 0)
          p.scales[(tile * kBlock + row) * (D / kGroup) + (lane * CPL) / kGroup] = (uint8_t)sc;
      }
    }
  }
}

// ---- element-wise encoder (pqkv_encode) ----
template <int CODE>
__global__ void encode_kernel(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    uint32_t c;
    if constexpr (CODE == PQKV_DTYPE_FP4_E2M1)
      c = enc_e2m1x2(v, 0.f) & 0xFu;
    else
      c = enc_fp8x2<CODE>(v, 0.f) & 0xFFu;
    out[i] = (uint8_t)c;
  }
}

// ---- launchers --------------------------------------------------------------

// Launch as a programmatic dependent of the previous kernel on the stream (the
// kernels wait for it at entry, so only the launch overlaps).
template <typename... Args>
static cudaError_t launch_pdl(void (*kern)(Args...), dim3 grid, unsigned block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t launch_write(int kv_dtype, int in_dtype, int D, const WriteParams& p, cudaStream_t st) {
  if (p.T <= 0) return cudaSuccess;
  const bool bf = (in_dtype == PQKV_DTYPE_BF16);
  if (kv_dtype == PQKV_DTYPE_FP16 || kv_dtype == PQKV_DTYPE_BF16) {
    const long warps = (long)p.T * p.Hkv;
    const int grid = (int)((warps + 7) / 8);
    return D == 128 ? launch_pdl(write16_kernel<128>, dim3(grid), 256, st, p)
                    : launch_pdl(write16_kernel<64>, dim3(grid), 256, st, p);
  }
  // a warp owns the runs starting in a window of tpw tokens of one (head, K|V)
  WriteParams q = p;
  q.tpw = (p.T <= 8192) ? 1 : 32;
  const dim3 grid((unsigned)((p.T + 4 * q.tpw - 1) / (4 * q.tpw)), (unsigned)p.Hkv, 2u);
#define PQKV_W8(F, DD, B) \
  if (kv_dtype == F && D == DD && bf == B) return launch_pdl(write_fp8_kernel<F, DD, B>, grid, 128, st, q);
  PQKV_W8(PQKV_DTYPE_FP8_E4M3, 128, true)
  PQKV_W8(PQKV_DTYPE_FP8_E4M3, 128, false)
  PQKV_W8(PQKV_DTYPE_FP8_E4M3, 64, true)
  PQKV_W8(PQKV_DTYPE_FP8_E4M3, 64, false)
  PQKV_W8(PQKV_DTYPE_FP8_E5M2, 128, true)
  PQKV_W8(PQKV_DTYPE_FP8_E5M2, 128, false)
  PQKV_W8(PQKV_DTYPE_FP8_E5M2, 64, true)
  PQKV_W8(PQKV_DTYPE_FP8_E5M2, 64, false)
#undef PQKV_W8
  if (kv_dtype == PQKV_DTYPE_FP4_E2M1) {
    if (D == 128)
      return bf ? launch_pdl(write_fp4_kernel<128, true>, grid, 128, st, q)
                : launch_pdl(write_fp4_kernel<128, false>, grid, 128, st, q);
    return bf ? launch_pdl(write_fp4_kernel<64, true>, grid, 128, st, q)
              : launch_pdl(write_fp4_kernel<64, false>, grid, 128, st, q);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_encode(int code_dtype, const float* x, int64_t n, uint8_t* out, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  switch (code_dtype) {
    case PQKV_DTYPE_FP8_E4M3: encode_kernel<PQKV_DTYPE_FP8_E4M3><<<grid, 256, 0, st>>>(x, n, out); break;
    case PQKV_DTYPE_FP8_E5M2: encode_kernel<PQKV_DTYPE_FP8_E5M2><<<grid, 256, 0, st>>>(x, n, out); break;
    case PQKV_DTYPE_FP4_E2M1: encode_kernel<PQKV_DTYPE_FP4_E2M1><<<grid, 256, 0, st>>>(x, n, out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pqkv
