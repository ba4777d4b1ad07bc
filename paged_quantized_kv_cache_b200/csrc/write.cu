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
#include <cfloat>

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

// x / d rounded to nearest even, for d a positive E4M3 value and r = 1 / d
// rounded to nearest (__frcp_rn): the product x r is corrected once by its
// residual x - d (x r), which an FMA computes exactly (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Develop. 34(1), 1990). The sign of a zero result is not kept;
// the encoder takes signs from x. The write's codes built on it are checked
// bit for bit against the oracle's IEEE division for every bf16 and fp16 input
// value and every E4M3 group scale that can occur together (tests).
__device__ __forceinline__ float div_by_scale(float x, float d, float r) {
  const float q0 = __fmul_rn(x, r);
  const float e = __fmaf_rn(-q0, d, x);
  return __fmaf_rn(e, r, q0);
}

// 16 quotients -> 16 E2M1 codes (channel 2i in the low nibble of byte i), the
// sign bit of each code taken from its input x (so that -0 and negative values
// rounding to zero keep their sign).
__device__ __forceinline__ uint2 e2m1_codes16(const float (&x)[16], float d, float r) {
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t c = 0, sg = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = x[8 * h + 2 * k], b = x[8 * h + 2 * k + 1];
      uint32_t byte;
      asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
          : "=r"(byte)
          : "f"(fabsf(div_by_scale(b, d, r))), "f"(fabsf(div_by_scale(a, d, r))));
      c |= byte << (8 * k);
      sg |= ((__float_as_uint(a) >> 31) << (8 * k + 3)) | ((__float_as_uint(b) >> 31) << (8 * k + 7));
    }
    w[h] = c | sg;
  }
  return make_uint2(w[0], w[1]);
}

// Lane layout: lane l takes the 16 channels of group g = l % GPL (GPL = D / 16
// groups per token) for block rows tl, tl + TL, ... (tl = l / GPL, TL = 32 /
// GPL): a token-group's absmax, scale and codes stay in one lane, and the two
// rows of a V token pair (r, r ^ 1) sit in lanes l and l ^ GPL.
// Four CTAs per SM (at most 128 registers a thread): the kernel is bound by
// instruction issue, and 16 warps per SM hide more latency than 12.
template <int D, bool INBF16>
__global__ void __launch_bounds__(128, 4) write_fp4_kernel(const WriteParams p) {
  // inputs may come from the previous kernel; let the next one start launching
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int GPL = D / kGroup;    // groups per token: 8 or 4
  constexpr int TL = 32 / GPL;       // lanes per group: 4 or 8
  constexpr int TPL = kBlock / TL;   // block rows per lane: 4 or 2
  constexpr int PREC = INBF16 ? 8 : 11;  // significant bits of an input value
  __shared__ float s_norm[4][D];
  __shared__ int s_oc[4][kOutSlots];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane % GPL, tl = lane / GPL;
  const int win = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, kv = blockIdx.z;
  const int t = win * p.tpw + lane;
  uint32_t starts = run_starts(p, t, lane < p.tpw, h == 0 && kv == 0);
  while (starts) {
    const int i0 = __ffs(starts) - 1;
    starts &= starts - 1;
    const int ts = win * p.tpw + i0;
    const int s0 = p.slots[ts];
    const int n = run_length(p, ts, s0, lane);
    const int blk = s0 >> 4, off0 = s0 & 15;
    const size_t tile = ((size_t)blk * p.Hkv + h) * 2 + kv;  // (block, head, K|V) index
    const auto* x = reinterpret_cast<const uint16_t*>(kv ? p.v : p.k);
    // this lane's rows of the run (rows outside it read as zeros)
    float xs[TPL][16];
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int r = tl + TL * i, j = r - off0;
      uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
      if (j >= 0 && j < n) {
        const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)(ts + j) * p.Hkv + h) * D + kGroup * g);
        u0 = __ldg(src);
        u1 = __ldg(src + 1);
      }
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if constexpr (INBF16) {
          xs[i][2 * k] = __uint_as_float(w[k] << 16);
          xs[i][2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        } else {
          xs[i][2 * k] = __half2float(__ushort_as_half((unsigned short)(w[k] & 0xFFFFu)));
          xs[i][2 * k + 1] = __half2float(__ushort_as_half((unsigned short)(w[k] >> 16)));
        }
      }
    }
    uint8_t* idxp = p.oidx + tile * kIdxStride;
    int oc[kOutSlots];  // outlier channels, ascending (>= D: empty)
    if (off0 == 0) {
      // step 1: channel norms (L-inf over the run's tokens), the same on every
      // lane of a group
      float nrm[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        nrm[c] = fabsf(xs[0][c]);
#pragma unroll
        for (int i = 1; i < TPL; ++i) nrm[c] = fmaxf(nrm[c], fabsf(xs[i][c]));
      }
#pragma unroll
      for (int o = GPL; o < 32; o <<= 1)
#pragma unroll
        for (int c = 0; c < 16; ++c) nrm[c] = fmaxf(nrm[c], __shfl_xor_sync(kFull, nrm[c], o));
      // step 2: mu + 3.2 sigma of the D norms, in fp64 as the channel-order sums
      // S1 = sum n, S2 = sum n^2. Norms are input values (PREC significant
      // bits); when the nonzero ones span at most 23 - PREC binades, every
      // partial sum of n and of n^2 is exact in fp64 (< 2^53 units of the
      // smallest term), so any order of summation gives the channel-order
      // result and the lanes add theirs in a tree. Otherwise: channel order.
      float mx = 0.f, mn = FLT_MAX;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        mx = fmaxf(mx, nrm[c]);
        mn = fminf(mn, nrm[c] > 0.f ? nrm[c] : FLT_MAX);
      }
#pragma unroll
      for (int o = 1; o < GPL; o <<= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
      }
      const bool exact = (mx == 0.f) || (mn >= FLT_MIN && ilogbf(mx) - ilogbf(mn) <= 23 - PREC);
      double s1 = 0.0, s2 = 0.0;
      if (exact) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const double v = (double)nrm[c];
          s1 = __dadd_rn(s1, v);
          s2 = __dadd_rn(s2, __dmul_rn(v, v));
        }
#pragma unroll
        for (int o = 1; o < GPL; o <<= 1) {
          s1 = __dadd_rn(s1, __shfl_xor_sync(kFull, s1, o));
          s2 = __dadd_rn(s2, __shfl_xor_sync(kFull, s2, o));
        }
      } else {
        if (tl == 0)
#pragma unroll
          for (int c = 0; c < 16; ++c) s_norm[warp][kGroup * g + c] = nrm[c];
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
        s1 = __shfl_sync(kFull, acc, 0);
        s2 = __shfl_sync(kFull, acc, 1);
        __syncwarp();
      }
      const double mu = __ddiv_rn(s1, (double)D);
      double var = __dsub_rn(__ddiv_rn(s2, (double)D), __dmul_rn(mu, mu));
      if (var < 0.0) var = 0.0;
      const double thr = __dadd_rn(mu, __dmul_rn(3.2, __dsqrt_rn(var)));
      uint32_t cand = 0;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if ((double)nrm[c] >= thr) cand |= 1u << c;
      // candidates of the groups before this lane's (a scan within the GPL lanes of a row)
      int incl = __popc(cand);
#pragma unroll
      for (int o = 1; o < GPL; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (g >= o) incl += v;
      }
      const int before = incl - __popc(cand);
      int total = __popc(cand);
#pragma unroll
      for (int o = 1; o < GPL; o <<= 1) total += __shfl_xor_sync(kFull, total, o);
      if (total <= kOutSlots) {
        // all candidates, in channel order
        if (tl == 0) {
          int k = before;
          uint32_t m = cand;
          while (m) {
            const int c = __ffs(m) - 1;
            m &= m - 1;
            s_oc[warp][k++] = kGroup * g + c;
          }
        }
        if (lane == 0)
          for (int k = total; k < kOutSlots; ++k) s_oc[warp][k] = 0xFF;
        __syncwarp();
#pragma unroll
        for (int r = 0; r < kOutSlots; ++r) oc[r] = s_oc[warp][r];
        __syncwarp();
      } else {
        // keep 4: largest norm first, ties to the lower channel; then ascending
#pragma unroll
        for (int r = 0; r < kOutSlots; ++r) {
          float bv = -1.f;
          int bc = 0x7FFFFFFF;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (((cand >> c) & 1u) && nrm[c] > bv) {
              bv = nrm[c];
              bc = kGroup * g + c;
            }
#pragma unroll
          for (int o = 1; o < GPL; o <<= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int occ = __shfl_xor_sync(kFull, bc, o);
            if (ov > bv || (ov == bv && occ < bc)) {
              bv = ov;
              bc = occ;
            }
          }
          oc[r] = bc;  // a candidate exists in every round (more than 4 of them)
          if ((bc >> 4) == g) cand &= ~(1u << (bc & 15));
        }
#pragma unroll
        for (int a2 = 1; a2 < kOutSlots; ++a2)
#pragma unroll
          for (int b2 = kOutSlots - 1; b2 >= a2; --b2)
            if (oc[b2 - 1] > oc[b2]) {
              const int tmp = oc[b2];
              oc[b2] = oc[b2 - 1];
              oc[b2 - 1] = tmp;
            }
      }
      if (lane == 0) {
        reinterpret_cast<uint32_t*>(idxp)[0] =
            (uint32_t)oc[0] | ((uint32_t)oc[1] << 8) | ((uint32_t)oc[2] << 16) | ((uint32_t)oc[3] << 24);
        reinterpret_cast<uint32_t*>(idxp)[1] = 0xFFFFFFFFu;
      }
    } else {
      const uint32_t lo = *reinterpret_cast<const uint32_t*>(idxp);
#pragma unroll
      for (int r = 0; r < kOutSlots; ++r) oc[r] = (lo >> (8 * r)) & 0xFF;
    }
    // step 3a: the fp16 outlier buffer, lane (row, slot) for 8 rows at a time,
    // read again from the input (the values are in L1/L2)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = (lane >> 2) + 8 * half, slot = lane & 3, j = r - off0;
      if (j >= 0 && j < n) {
        int c = 0xFF;
#pragma unroll
        for (int k = 0; k < kOutSlots; ++k)
          if (k == slot) c = oc[k];
        unsigned short hv = 0;
        if (c < D) {
          const uint16_t raw = x[((size_t)(ts + j) * p.Hkv + h) * D + c];
          hv = INBF16 ? __half_as_ushort(__float2half_rn(__uint_as_float((uint32_t)raw << 16))) : raw;
        }
        reinterpret_cast<unsigned short*>(p.oval)[(tile * kBlock + r) * kOutSlots + slot] = hv;
      }
    }
    // outlier channels of this lane's group get code 0 and stay out of the
    // group absmax: zero them
    uint32_t om = 0;
#pragma unroll
    for (int r = 0; r < kOutSlots; ++r)
      if (oc[r] < D && (oc[r] >> 4) == g) om |= 1u << (oc[r] & 15);
    if (om) {
#pragma unroll
      for (int i = 0; i < TPL; ++i)
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if ((om >> c) & 1u) xs[i][c] = 0.f;
    }
    // step 3b: per row, E4M3 group scale and E2M1 codes
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int r = tl + TL * i, j = r - off0;
      const bool act = j >= 0 && j < n;
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) a = fmaxf(a, fabsf(xs[i][c]));
      const uint32_t sc = enc_fp8x2<PQKV_DTYPE_FP8_E4M3>(__fdiv_rn(a, 6.0f), 0.f) & 0xFFu;
      const float sd = e4m3_value(sc);
      uint2 codes = make_uint2(0u, 0u);
      if (sd > 0.f) codes = e2m1_codes16(xs[i], sd, __frcp_rn(sd));
      if (act) p.scales[(tile * kBlock + r) * GPL + g] = (uint8_t)sc;
      if (kv == 0) {
        // K: one row per token
        if (act) *reinterpret_cast<uint2*>(p.cache + (tile * kBlock + r) * (D / 2) + 8 * g) = codes;
      } else {
        // V: a byte holds one channel of a token pair (even row in the low
        // nibble); the partner row sits in lane ^ GPL. A pair split by the
        // run's ends keeps the other row's nibbles.
        const uint32_t o0 = __shfl_xor_sync(kFull, codes.x, GPL);
        const uint32_t o1 = __shfl_xor_sync(kFull, codes.y, GPL);
        const bool pact = (r ^ 1) - off0 >= 0 && (r ^ 1) - off0 < n;
        const bool even = (r & 1) == 0;
        if (act && (even || !pact)) {
          const uint32_t e0 = even ? codes.x : o0, e1 = even ? codes.y : o1;  // even row's codes
          const uint32_t d0 = even ? o0 : codes.x, d1 = even ? o1 : codes.y;  // odd row's codes
          // channel 2k of the even row -> low nibble, of the odd row -> high nibble
          auto spread = [](uint32_t ev, uint32_t od) -> uint4 {
            const uint32_t lo_e = ev & 0x0F0F0F0Fu, hi_e = (ev >> 4) & 0x0F0F0F0Fu;
            const uint32_t lo_o = (od & 0x0F0F0F0Fu) << 4, hi_o = od & 0xF0F0F0F0u;
            const uint32_t ce = lo_e | lo_o;  // channels 0, 2, 4, 6 (bytes)
            const uint32_t co = hi_e | hi_o;  // channels 1, 3, 5, 7
            return make_uint4(prmt(ce, co, 0x5140u), prmt(ce, co, 0x7362u), 0u, 0u);
          };
          const uint4 lo8 = spread(e0, d0), hi8 = spread(e1, d1);
          uint4 out = make_uint4(lo8.x, lo8.y, hi8.x, hi8.y);
          const int pr = (r < 8) ? (r & ~1) : (((r - 8) & ~1) + 1);
          const int cb = kGroup * g;
          uint4* dst = reinterpret_cast<uint4*>(p.cache + (tile * kBlock + 8 * (cb / (D / 2)) + pr) * (D / 2) +
                                                cb % (D / 2));
          if (!pact) {  // only this row: keep the partner's nibbles
            const uint4 cur = *dst;
            const uint32_t keep = even ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
            out.x = (cur.x & keep) | (out.x & ~keep);
            out.y = (cur.y & keep) | (out.y & ~keep);
            out.z = (cur.z & keep) | (out.z & ~keep);
            out.w = (cur.w & keep) | (out.w & ~keep);
          }
          *dst = out;
        }
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
