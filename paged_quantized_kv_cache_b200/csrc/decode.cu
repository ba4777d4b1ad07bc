// decode.cu -- the paged decode-attention kernel (see decode.cuh for the design).
#include <atomic>
#include <cfloat>

#include "decode.cuh"

namespace pqkv {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kNegInf = -INFINITY;
// The running max m is only moved (and O, l rescaled) when a block's max
// exceeds it by more than this many log2 units, so most blocks skip the
// rescale; probabilities then stay below 2^kLazy, well inside f16 / bf16.
// FP4 multiplies P by E4M3 group scales (<= 448) in f16, so it keeps P <= 16.
template <int KVF>
constexpr float lazy_of() { return KVF == PQKV_DTYPE_FP4_E2M1 ? 4.f : 8.f; }

// Zero the low (token t0) / high (token t0 + 1) half of a packed pair when the
// token lies past the end of the sequence (its bytes may hold anything).
__device__ __forceinline__ uint32_t mask_pair(uint32_t v, int t0, int valid) {
  if (t0 >= valid) v &= 0xFFFF0000u;
  if (t0 + 1 >= valid) v &= 0x0000FFFFu;
  return v;
}

__device__ __forceinline__ uint32_t f16x2_from(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 2^x with the hardware approximation (relative error ~2^-22, denormal results flushed).
__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Element offset of the q / out row of MMA column c of KV head h of sequence
// b: q and out are [B][k][Hq][D], column c = (token q0 + c / Gh, head c % Gh).
__device__ __forceinline__ size_t col_row(int b, int h, int c, int k, int q0, int Gh, int Hq, int D) {
  return ((size_t)(b * k + q0 + c / Gh) * Hq + (size_t)h * Gh + c % Gh) * D;
}

template <bool QBF16>
__device__ __forceinline__ float q_at(const void* q, size_t i) {
  if constexpr (QBF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]);
  else
    return __half2float(reinterpret_cast<const __half*>(q)[i]);
}

template <bool QBF16>
__device__ __forceinline__ void store_out(void* out, size_t i, float v) {
  if constexpr (QBF16)
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<__half*>(out)[i] = __float2half_rn(v);
}

// out[i], out[i + 1] = a, b in one 4-byte store (i even).
template <bool QBF16>
__device__ __forceinline__ void store_out2(void* out, size_t i, float a, float b) {
  if constexpr (QBF16)
    *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(out) + i) = __floats2bfloat162_rn(a, b);
  else
    *reinterpret_cast<__half2*>(reinterpret_cast<__half*>(out) + i) = __floats2half2_rn(a, b);
}

// Four E4M3 codes -> f16x2 of bytes (0,1) and (2,3) by the hardware conversion.
__device__ __forceinline__ void dec4_e4m3_cvt(uint32_t r, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(r));
}

// Four FP8 codes of a word -> f16x2 of bytes (0,1) and of bytes (2,3), exact.
// E5M2 codes are the high byte of the binary16 of the same value, so they are
// placed, not converted; E4M3 codes go through the hardware conversion (placing
// their bits too, as the binary16 of value x 2^-8 with three integer
// operations per pair, measured 20% slower per decode: the kernel is bound by
// instruction issue, not by the conversions).
template <int KVF>
__device__ __forceinline__ void dec4(uint32_t r, uint32_t& lo, uint32_t& hi) {
  if constexpr (KVF == PQKV_DTYPE_FP8_E5M2) {
    lo = prmt(r, 0u, 0x1404u);
    hi = prmt(r, 0u, 0x3424u);
  } else {
    dec4_e4m3_cvt(r, lo, hi);
  }
}

// Per-lane shared-memory offsets (bytes, within a stage) of the ldmatrix rows
// of one block: K reads of k-step group i and V reads of m-tile group i. The
// swizzle depends on the lane, so these are computed once per kernel.
template <int KVF, int D>
struct LdsmOffsets {
  using Gm = DecodeGeom<KVF, D>;
  // 16-bit: one x4 per 16 head dims; FP8: per 32 dims; FP4: per 64 dims
  static constexpr int kN = Gm::k16 ? D / 16 : (Gm::kFp8 ? D / 32 : D / 64);
  uint32_t k[kN], v[kN];
  __device__ __forceinline__ explicit LdsmOffsets(int lane) {
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int i = 0; i < kN; ++i) {
      if constexpr (Gm::k16) {
        k[i] = Gm::off(((mi & 1) << 3) + ri, (2 * i + (mi >> 1)) * 16);
        v[i] = Gm::off(16 + ((mi >> 1) << 3) + ri, (2 * i + (mi & 1)) * 16);
      } else if constexpr (Gm::kFp8) {
        k[i] = Gm::off(((mi & 1) << 3) + ri, (2 * i + (mi >> 1)) * 16);
        v[i] = Gm::off(16 + ((mi & 1) << 3) + ri, (2 * i + (mi >> 1)) * 16);
      } else {
        // V: matrix mi of load i is m-tile c = 4i + mi, the 8 pair rows of
        // its half of the channels at the 16-byte column of its 16 channels
        const int c = 4 * i + mi;
        k[i] = Gm::off(((mi & 1) << 3) + ri, (2 * i + (mi >> 1)) * 16);
        v[i] = Gm::off(16 + 8 * (c / (D / 32)) + ri, 16 * (c % (D / 32)));
      }
    }
  }
};

// Row `rr` (0..15) of output m-tile `mt` -> head-dimension index. The order
// of d inside a tile follows how each format's dequantization lays out the
// V^T fragment (see block_pv).
template <int KVF>
__device__ __forceinline__ int dmap(int mt, int rr) {
  if constexpr (KVF == PQKV_DTYPE_FP16 || KVF == PQKV_DTYPE_BF16) {
    return 16 * mt + rr;
  } else {
    // FP8, FP4: tile c covers [16c, 16c + 16): row g -> 16c + 2g, row g + 8 -> 16c + 2g + 1
    return 16 * mt + 2 * (rr & 7) + (rr >> 3);
  }
}

// FP4 outlier channels: per-warp state carried from block to block. The
// outlier channels of consecutive blocks of one KV head usually agree, so the
// query fragment at the K outlier channels and the V outlier product are kept
// in registers while the channel set stays the same; the V product goes to the
// shared-memory accumulator of outlier channels only when the set changes or
// the piece ends.
template <int NT>
struct OutlierState {
  static constexpr uint32_t kNone = 0xFEFEFEFEu;  // no valid channel byte (they are < 128 or 0xFF)
  uint32_t kidx;        // K outlier channels the cached query fragments belong to
  uint32_t kq[NT];      // query fragments (B of the K outlier MMA), per column tile
  uint32_t vidx;        // V outlier channels vacc belongs to
  float vacc[NT][4];    // V outlier product (rows = slots, lanes g < 4) not yet flushed
  __device__ __forceinline__ void reset() {
    kidx = vidx = kNone;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      kq[nt] = 0;
      vacc[nt][0] = vacc[nt][1] = vacc[nt][2] = vacc[nt][3] = 0.f;
    }
  }
  // add vacc into the accumulator of outlier channels and clear it
  template <int STRIDE>
  __device__ __forceinline__ void flush(float* oext, int lane, int D) {
    const int g = lane >> 2, qd = lane & 3;
    if (vidx != kNone && g < 4) {
      const int dch = (vidx >> (8 * g)) & 0xFF;
      if (dch < D) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          oext[(8 * nt + 2 * qd) * STRIDE + dch] += vacc[nt][0];
          oext[(8 * nt + 2 * qd + 1) * STRIDE + dch] += vacc[nt][1];
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) vacc[nt][0] = vacc[nt][1] = vacc[nt][2] = vacc[nt][3] = 0.f;
  }
};

// ---------------------------------------------------------------------------
// S^T (16 tokens x 8 NT query rows) += K Q^T for one block in shared memory.
// Lane (g, qd) ends with rows (tokens) g, g + 8 and columns 8nt + 2qd, 8nt +
// 2qd + 1 of each column tile nt; the K fragments are dequantized once for all.
// ---------------------------------------------------------------------------
template <int KVF, int D, int NT>
__device__ __forceinline__ void block_scores(uint32_t tb, const uint8_t* side,
                                             const uint32_t (&qf)[NT][D / 16][2], const uint16_t* wq,
                                             const LdsmOffsets<KVF, D>& lo, int lane, float (&sc)[NT][4],
                                             OutlierState<NT>& ost) {
  using Gm = DecodeGeom<KVF, D, NT>;
  constexpr int KT = D / 16;
  const int g = lane >> 2, qd = lane & 3;
  float se[NT][4], so[NT][4];  // two independent chains per column tile
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) se[nt][i] = so[nt][i] = 0.f;
  if constexpr (Gm::k16) {
    constexpr bool kBf = (KVF == PQKV_DTYPE_BF16);
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(tb + lo.k[kk], a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (kk & 1) mma16816<kBf>(so[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
        else mma16816<kBf>(se[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
      }
    }
  } else if constexpr (Gm::kFp8) {
    // ldmatrix on byte data: lane (g, qd) receives bytes 4qd..4qd+3 of a token
    // row's 16-byte chunk, i.e. 4 consecutive d of one k-step.
#pragma unroll
    for (int cp = 0; cp < KT / 2; ++cp) {
      uint32_t r0, r1, r2, r3;
      ldsm_x4(tb + lo.k[cp], r0, r1, r2, r3);
      uint32_t x0l, x0h, x1l, x1h, x2l, x2h, x3l, x3h;
      dec4<KVF>(r0, x0l, x0h);
      dec4<KVF>(r1, x1l, x1h);
      dec4<KVF>(r2, x2l, x2h);
      dec4<KVF>(r3, x3l, x3h);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma16816<false>(se[nt], x0l, x1l, x0h, x1h, qf[nt][2 * cp][0], qf[nt][2 * cp][1]);
        mma16816<false>(so[nt], x2l, x3l, x2h, x3h, qf[nt][2 * cp + 1][0], qf[nt][2 * cp + 1][1]);
      }
    }
  } else {
    // FP4: one 16-byte chunk = 32 d; lane (g, qd) receives the 8 codes
    // d = 32c + 8qd .. +7 of token rows g and g + 8 and multiplies them by the
    // token's E4M3 scale of group 2c + qd/2 (the product is exact in f16).
    constexpr int SPR = D / 16;  // scale bytes per token row
    // The scale of chunk c for this lane is byte 2c + qd/2 of the token's scale
    // row: pick it from whole words and broadcast it to (s, s) in f16.
    uint32_t sa2[D / 32], sb2[D / 32];
    {
      const int a = qd >> 1;
      const uint32_t sel = (uint32_t)(a | (a << 4) | ((a + 2) << 8) | ((a + 2) << 12));
      const uint32_t* ra = reinterpret_cast<const uint32_t*>(side + g * SPR);
      const uint32_t* rb = reinterpret_cast<const uint32_t*>(side + (g + 8) * SPR);
#pragma unroll
      for (int w = 0; w < SPR / 4; ++w) {  // word w = groups 4w..4w+3 = chunks 2w, 2w+1
        dec4_e4m3_cvt(prmt(ra[w], 0u, sel), sa2[2 * w], sa2[2 * w + 1]);
        dec4_e4m3_cvt(prmt(rb[w], 0u, sel), sb2[2 * w], sb2[2 * w + 1]);
      }
    }
#pragma unroll
    for (int cp = 0; cp < D / 64; ++cp) {
      uint32_t r0, r1, r2, r3;
      ldsm_x4(tb + lo.k[cp], r0, r1, r2, r3);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = 2 * cp + e;
        const uint32_t ra = e ? r2 : r0, rb = e ? r3 : r1;
        const __half2 sa = *reinterpret_cast<const __half2*>(&sa2[c]);
        const __half2 sb = *reinterpret_cast<const __half2*>(&sb2[c]);
        uint32_t ha[4], hb[4];
        dec_e2m1x8(ra, ha);
        dec_e2m1x8(rb, hb);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          __half2 xa = __hmul2(*reinterpret_cast<__half2*>(&ha[i]), sa);
          __half2 yb = __hmul2(*reinterpret_cast<__half2*>(&hb[i]), sb);
          ha[i] = *reinterpret_cast<uint32_t*>(&xa);
          hb[i] = *reinterpret_cast<uint32_t*>(&yb);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma16816<false>(se[nt], ha[0], hb[0], ha[1], hb[1], qf[nt][2 * c][0], qf[nt][2 * c][1]);
          mma16816<false>(so[nt], ha[2], hb[2], ha[3], hb[3], qf[nt][2 * c + 1][0], qf[nt][2 * c + 1][1]);
        }
      }
    }
    // outlier channels (their codes are 0): S^T += Kout (16 tokens x 4 slots) Qout^T.
    // Empty slots hold +0 values and get a zero query, so they add nothing.
    {
      const uint32_t kw = *reinterpret_cast<const uint32_t*>(side + Gm::kScaleBytes + Gm::kValBytes);  // K idx
      const uint32_t* kv = reinterpret_cast<const uint32_t*>(side + Gm::kScaleBytes);  // K vals [16][4] fp16
      if (kw != ost.kidx) {  // same for the whole warp
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t b0 = 0;
          if (qd < 2) {
            const int r0i = (kw >> (16 * qd)) & 0xFF, r1i = (kw >> (16 * qd + 8)) & 0xFF;
            const uint16_t* row = wq + (8 * nt + g) * Gm::kQStride;
            const uint32_t q0 = (r0i < D) ? row[r0i] : 0u;
            const uint32_t q1 = (r1i < D) ? row[r1i] : 0u;
            b0 = q0 | (q1 << 16);
          }
          ost.kq[nt] = b0;
        }
        ost.kidx = kw;
      }
      const uint32_t a0 = (qd < 2) ? kv[g * 2 + qd] : 0u;
      const uint32_t a1 = (qd < 2) ? kv[(g + 8) * 2 + qd] : 0u;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma16816<false>(so[nt], a0, a1, 0u, 0u, ost.kq[nt], 0u);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[nt][i] = se[nt][i] + so[nt][i];
}

// ---------------------------------------------------------------------------
// O^T (D x 8 NT query rows) += V^T P^T for one block. P^T arrives per column
// tile as two B fragments (hi and lo parts, P = P_hi + P_lo rounded to the
// operand type); the V fragments are dequantized once for all tiles.
// ---------------------------------------------------------------------------
template <int KVF, int D, int NT>
__device__ __forceinline__ void block_pv(uint32_t tb, const uint8_t* side, const LdsmOffsets<KVF, D>& lo, int lane,
                                         int valid, const uint32_t (&b0)[NT], const uint32_t (&b1)[NT],
                                         const uint32_t (&c0)[NT], const uint32_t (&c1)[NT],
                                         float (&acc)[NT][D / 16][4], float* oext, OutlierState<NT>& ost) {
  using Gm = DecodeGeom<KVF, D, NT>;
  constexpr int KT = D / 16;
  constexpr bool kBf = (KVF == PQKV_DTYPE_BF16);
  const int g = lane >> 2, qd = lane & 3;
  const int t0 = 2 * qd, t1 = 2 * qd + 8;
  // FP4 keeps P in f16 only (its tolerance allows it); the others add P_lo.
  constexpr bool kSplitP = !Gm::kFp4;
  auto mma_pv = [&](int nt, float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
    mma16816<kBf>(d, a0, a1, a2, a3, b0[nt], b1[nt]);
    if constexpr (kSplitP) mma16816<kBf>(d, a0, a1, a2, a3, c0[nt], c1[nt]);
  };
  if constexpr (Gm::k16) {
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(tb + lo.v[mt], a0, a1, a2, a3);
      if (valid < kBlock) {
        a0 = mask_pair(a0, t0, valid);
        a1 = mask_pair(a1, t0, valid);
        a2 = mask_pair(a2, t1, valid);
        a3 = mask_pair(a3, t1, valid);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_pv(nt, acc[nt][mt], a0, a1, a2, a3);
    }
  } else if constexpr (Gm::kFp8) {
    // ldmatrix.trans on byte data: lane (g, qd) receives d0 = 16c + 2g and d0 + 1
    // of tokens 2qd and 2qd + 1; one byte permute pairs the tokens per d.
#pragma unroll
    for (int cp = 0; cp < KT / 2; ++cp) {
      uint32_t r0, r1, r2, r3;
      ldsm_x4_t(tb + lo.v[cp], r0, r1, r2, r3);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t xa = prmt(e ? r2 : r0, 0u, 0x3120u);
        const uint32_t xb = prmt(e ? r3 : r1, 0u, 0x3120u);
        uint32_t a0, a1, a2, a3;
        dec4<KVF>(xa, a0, a1);
        dec4<KVF>(xb, a2, a3);
        if (valid < kBlock) {
          a0 = mask_pair(a0, t0, valid);
          a1 = mask_pair(a1, t0, valid);
          a2 = mask_pair(a2, t1, valid);
          a3 = mask_pair(a3, t1, valid);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_pv(nt, acc[nt][2 * cp + e], a0, a1, a2, a3);
      }
    }
  } else {
    // FP4: a V byte holds one channel of a token pair, so ldmatrix.trans of 8
    // pair rows hands lane (g, qd) the whole A fragment of m-tile c in one word:
    // d = 16c + 2g, 16c + 2g + 1 of tokens (2qd, 2qd + 1) and (2qd + 8, 2qd + 9).
    // m-tile c is scale group c, so the tokens' E4M3 group scales multiply P
    // (in f16: P <= 16, scale <= 448) instead of the codes.
    constexpr int SPR = D / 16;
    const uint8_t* vs = side + 16 * SPR;  // V scales [16][D/16]
    uint32_t sp[2][D / 16];               // (s(t, c), s(t + 1, c)), t = 2qd | 2qd + 8
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int ta = 2 * qd + 8 * hh;
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(vs + ta * SPR);
      const uint32_t* w1 = reinterpret_cast<const uint32_t*>(vs + (ta + 1) * SPR);
#pragma unroll
      for (int w = 0; w < SPR / 4; ++w) {
        dec4_e4m3_cvt(prmt(w0[w], w1[w], 0x5140u), sp[hh][4 * w], sp[hh][4 * w + 1]);
        dec4_e4m3_cvt(prmt(w0[w], w1[w], 0x7362u), sp[hh][4 * w + 2], sp[hh][4 * w + 3]);
      }
      if (valid < kBlock) {  // scales past the end may be NaN codes
#pragma unroll
        for (int c = 0; c < D / 16; ++c) sp[hh][c] = mask_pair(sp[hh][c], ta, valid);
      }
    }
#pragma unroll
    for (int i = 0; i < D / 64; ++i) {
      uint32_t r[4];
      ldsm_x4_t(tb + lo.v[i], r[0], r[1], r[2], r[3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 4 * i + e;
        uint32_t a[4];
        dec_e2m1x8(r[e], a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const __half2 p0 =
              __hmul2(*reinterpret_cast<const __half2*>(&b0[nt]), *reinterpret_cast<const __half2*>(&sp[0][c]));
          const __half2 p1 =
              __hmul2(*reinterpret_cast<const __half2*>(&b1[nt]), *reinterpret_cast<const __half2*>(&sp[1][c]));
          mma16816<false>(acc[nt][c], a[0], a[1], a[2], a[3], *reinterpret_cast<const uint32_t*>(&p0),
                          *reinterpret_cast<const uint32_t*>(&p1));
        }
      }
    }
    // outlier channels: Oext[n][idx_r] += (Vout^T (4 slots x 16 tokens) P^T)[r][n].
    // The result of slot r sits in lanes 4r..4r+3 (heads 2qd, 2qd+1); it stays
    // in registers while the block's V outlier channels match the previous
    // block's, and goes to the warp's shared-memory accumulator of outlier
    // channels (which follows O's rescaling and is folded into O when the piece
    // ends) when they change.
    {
      const uint32_t vw = *reinterpret_cast<const uint32_t*>(side + Gm::kScaleBytes + Gm::kValBytes + 8);  // V idx
      const uint16_t* vv = reinterpret_cast<const uint16_t*>(side + Gm::kScaleBytes + 128);    // V vals
      if (vw != ost.vidx) {  // same for the whole warp
        ost.template flush<Gm::kOStride>(oext, lane, D);
        ost.vidx = vw;
      }
      uint32_t a0 = 0, a2 = 0;
      if (g < 4) {
        a0 = (uint32_t)vv[t0 * 4 + g] | ((uint32_t)vv[(t0 + 1) * 4 + g] << 16);
        a2 = (uint32_t)vv[t1 * 4 + g] | ((uint32_t)vv[(t1 + 1) * 4 + g] << 16);
        if (valid < kBlock) {
          a0 = mask_pair(a0, t0, valid);
          a2 = mask_pair(a2, t1, valid);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_pv(nt, ost.vacc[nt], a0, 0u, a2, 0u);
    }
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Log-sum-exp merge of a split pair ("Flash-Decoding": the partial softmaxes of
// the pieces are combined as M = max_j m_j, L = sum_j l_j 2^(m_j - M),
// out = sum_j O_j 2^(m_j - M) / L, in fixed piece order) for all G columns of
// the pair (b, h) whose np >= 2 pieces start in chunk k0. Run by one warp: the
// warp whose piece completed the pair (see arrive_split), so results do not
// depend on which warp that is or on timing. It runs at the end of that warp's
// chunk, so it is written for latency: a group of 8 lanes per column, 4
// columns at a time; lane j of a group holds the (m, l) of pieces j, j + 8, ...
// (reduced over the group), and the outputs of kB pieces are loaded at once,
// the first kB together with the (m, l). For the usual np <= kB that is one
// round trip to L2 per 4 columns.
// ---------------------------------------------------------------------------
template <int D, bool QBF16>
__device__ __forceinline__ void merge_pair(const DecodeParams& p, int b, int h, int k0, int np, int lane) {
  constexpr int DL = D / 8;   // head dims per lane
  constexpr int V4 = DL / 4;  // float4 per lane and piece
  constexpr int kB = D == 128 ? 2 : 4;  // pieces whose outputs are loaded together
  const int G = p.G;
  const int j = lane & 7, gbase = lane & ~7;
  auto slot_base = [&](int i) {  // piece i (0-based) of the pair
    const int kk = k0 + i;
    return p.partials + (size_t)(i == 0 ? 2 * kk + 1 : 2 * kk) * p.slot_floats;
  };
  for (int n0 = 0; n0 < G; n0 += 4) {
    const int n = n0 + (lane >> 3), d0 = j * DL;
    const bool act = n < G;  // the same on the 8 lanes of a group
    float4 v[kB][V4];
    auto load_batch = [&](int c0) {
#pragma unroll
      for (int u = 0; u < kB; ++u)
#pragma unroll
        for (int q = 0; q < V4; ++q)
          v[u][q] = (act && c0 + u < np) ? __ldcg(reinterpret_cast<const float4*>(slot_base(c0 + u) + n * D + d0) + q)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    load_batch(0);
    // weights: lane j of the group takes pieces j, j + 8, ...
    float mA = kNegInf, lA = 0.f;
    if (act && j < np) {
      mA = __ldcg(slot_base(j) + G * D + n);
      lA = __ldcg(slot_base(j) + G * D + G + n);
    }
    float M = mA;
    if (act)
      for (int i = j + 8; i < np; i += 8) M = fmaxf(M, __ldcg(slot_base(i) + G * D + n));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    const float wA = (M == kNegInf || j >= np) ? 0.f : exp2f(mA - M);  // weight of piece j
    float L = wA * lA;
    if (act && M != kNegInf)
      for (int i = j + 8; i < np; i += 8)
        L += exp2f(__ldcg(slot_base(i) + G * D + n) - M) * __ldcg(slot_base(i) + G * D + G + n);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) L += __shfl_xor_sync(kFull, L, o);
    // outputs: pieces in order
    float acc[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < np; c0 += kB) {
      if (c0 > 0) load_batch(c0);
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int i = c0 + u;
        float w = __shfl_sync(kFull, wA, gbase | (i & 7));  // piece i < 8: held by lane i of the group
        if (i >= 8) w = (!act || M == kNegInf) ? 0.f : exp2f(__ldcg(slot_base(i) + G * D + n) - M);
        if (i < np) {
#pragma unroll
          for (int q = 0; q < V4; ++q) {
            acc[4 * q + 0] += w * v[u][q].x;
            acc[4 * q + 1] += w * v[u][q].y;
            acc[4 * q + 2] += w * v[u][q].z;
            acc[4 * q + 3] += w * v[u][q].w;
          }
        }
      }
    }
    if (act) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const size_t orow = col_row(b, h, n, p.k, p.q0, p.Gh, p.Hq, D) + d0;
#pragma unroll
      for (int e = 0; e < DL; ++e) store_out<QBF16>(p.out, orow + e, acc[e] * inv);
    }
  }
}

// Arrival words. counters[k0] (k0 = the chunk where a split pair starts) holds
// the launch's tag in its high 40 bits and the pieces of the pair counted so
// far in its low 24. A word whose tag is not this launch's (left by an earlier
// or aborted launch, or whatever the workspace held) reads as zero pieces, so
// the workspace needs no clearing. Adds n pieces (lane 0 only; the warp's
// partials are made visible first) and returns the count after the add. Pieces
// of one pair never wait on one another; the bounded loop only retries when
// another update got in between.
__device__ __forceinline__ unsigned long long count_pieces(const DecodeParams& p, int k0, int n) {
  __threadfence();  // this warp's partials are visible before the arrivals count
  unsigned long long* w = p.counters + k0;
  const unsigned long long tag = (unsigned long long)p.epoch << 24;
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(w);
  for (int it = 0; it < 4096; ++it) {
    const unsigned long long have = ((cur >> 24) == p.epoch) ? (cur & 0xFFFFFFull) : 0ull;
    const unsigned long long prev = atomicCAS(w, cur, tag | (have + (unsigned long long)n));
    if (prev == cur) return have + (unsigned long long)n;
    cur = prev;
  }
  raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
  return 0;
}

// A warp has written its piece of a short pair (all lanes' stores done): count
// it and tell whether it was the last one (its warp then merges the pair).
__device__ __forceinline__ bool arrive_split(const DecodeParams& p, int k0, int np, int lane) {
  int last = 0;
  if (lane == 0) {
    last = count_pieces(p, k0, 1) == (unsigned long long)np;
    if (last) __threadfence();  // order the reads of the other pieces after the count
  }
  return __shfl_sync(kFull, last, 0) != 0;
}

// Count n pieces of a long pair that this warp has written (all lanes' stores
// done). The pair is merged by the warps that own its output columns, which
// poll the word (wait_pieces).
__device__ __forceinline__ void publish_pieces(const DecodeParams& p, int k0, int n, int lane) {
  if (lane == 0 && n > 0) count_pieces(p, k0, n);
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of one output column (query row n of the pair (b, h)) over
// the np > kMergeInKernel pieces of a long split pair (same formula as
// merge_pair), by one warp: the (m, l) of every piece with lanes over pieces,
// then the outputs with lanes over head dims, pieces in order, the loads of up
// to kBatch pieces issued before they are folded in (the first batch together
// with the (m, l) loads).
// ---------------------------------------------------------------------------
template <int D, bool QBF16, int kBatch>
__device__ __forceinline__ void merge_column(const DecodeParams& p, int b, int h, int n, int k0, int np, int lane) {
  constexpr int DPL = D / 32;  // head dims per lane
  const int G = p.G;
  auto slot_base = [&](int i) {  // piece i (0-based) of the pair
    const int kk = k0 + i;
    return p.partials + (size_t)(i == 0 ? 2 * kk + 1 : 2 * kk) * p.slot_floats;
  };
  float v[kBatch][DPL];
  auto load_batch = [&](int i0) {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u;
      if (i < np) {
        const float* bs = slot_base(i) + n * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 t = __ldcg(reinterpret_cast<const float4*>(bs));
          v[u][0] = t.x; v[u][1] = t.y; v[u][2] = t.z; v[u][3] = t.w;
        } else {
          const float2 t = __ldcg(reinterpret_cast<const float2*>(bs));
          v[u][0] = t.x; v[u][1] = t.y;
        }
      }
    }
  };
  load_batch(0);
  float mi[4], li[4];  // pieces lane, lane + 32, lane + 64, lane + 96
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = lane + 32 * r;
    mi[r] = kNegInf;
    li[r] = 0.f;
    if (i < np) {
      const float* bs = slot_base(i);
      mi[r] = __ldcg(bs + G * D + n);
      li[r] = __ldcg(bs + G * D + G + n);
    }
  }
  float M = fmaxf(fmaxf(mi[0], mi[1]), fmaxf(mi[2], mi[3]));
  for (int i = lane + 128; i < np; i += 32) M = fmaxf(M, __ldcg(slot_base(i) + G * D + n));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
  float wr[4];
  float L = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    wr[r] = (M == kNegInf || mi[r] == kNegInf) ? 0.f : exp2f(mi[r] - M);
    L += wr[r] * li[r];
  }
  for (int i = lane + 128; i < np; i += 32) {
    const float* bs = slot_base(i);
    L += (M == kNegInf) ? 0.f : exp2f(__ldcg(bs + G * D + n) - M) * __ldcg(bs + G * D + G + n);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(kFull, L, o);
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int i0 = 0; i0 < np; i0 += kBatch) {
    if (i0 > 0) load_batch(i0);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u;
      if (i < np) {  // the same on every lane
        float w;
        if (i < 128) {
          const int r = i >> 5;
          w = __shfl_sync(kFull, r == 0 ? wr[0] : r == 1 ? wr[1] : r == 2 ? wr[2] : wr[3], i & 31);
        } else {
          w = (M == kNegInf) ? 0.f : exp2f(__ldcg(slot_base(i) + G * D + n) - M);
        }
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] += w * v[u][e];
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const size_t orow = col_row(b, h, n, p.k, p.q0, p.Gh, p.Hq, D) + lane * DPL;
#pragma unroll
  for (int e = 0; e < DPL; ++e) store_out<QBF16>(p.out, orow + e, acc[e] * inv);
}

// Wait until the arrival word of the pair whose first unit is k0 shows all its
// np pieces (lane 0 polls it, sleeping between polls), giving up after the
// wait limit. The pieces come from other warps of the same persistent grid,
// all resident, which never wait for this one, so the wait ends unless one of
// them gave up itself.
__device__ __forceinline__ bool wait_pieces(const DecodeParams& p, int k0, int np, int lane) {
  int ok = 0;
  if (lane == 0) {
    const volatile unsigned long long* w = p.counters + k0;
    const unsigned long long want = ((unsigned long long)p.epoch << 24) | (unsigned long long)np;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      if (*w == want) {
        ok = 1;
        break;
      }
      if (globaltimer_ns() - t0 > p.timeout_ns) break;
      __nanosleep(128);
    }
    __threadfence();  // order the reads of the pieces after the count
  }
  return __shfl_sync(kFull, ok, 0) != 0;
}

template <int KVF, int D, bool QBF16, int NT>
__global__ void __launch_bounds__(DecodeGeom<KVF, D, NT>::kWarps * 32, 1)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p) {
  using Gm = DecodeGeom<KVF, D, NT>;
  using Sm = DecodeSmem<KVF, D, NT>;
  constexpr int NC = Gm::kCols;  // MMA columns (query rows of one KV head) per warp
  constexpr int NW = Gm::kWarps;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // inputs may come from the previous kernel
  constexpr int NS = Gm::kStages;
  constexpr int KT = D / 16;  // k-steps of QK^T and m-tiles of PV
  constexpr bool kBf16Mma = (KVF == PQKV_DTYPE_BF16);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* tiles = smem;
  uint8_t* sides = tiles + Sm::kTilesBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sides + Sm::kSideBytes);
  uint16_t* qcopy = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(bars) + Sm::kBarBytes);
  float* oext_all = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(qcopy) + Sm::kQBytes);
  int* P = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(oext_all) + Sm::kOextBytes);
  __shared__ int warp_sums[NW];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int B = p.B, Hkv = p.Hkv, G = p.G, Hq = p.Hq;
  const int g = lane >> 2, qd = lane & 3;
  // multi-query: positions at the end of the sequence hidden from this lane's
  // columns n = 8nt + 2qd + c (query token q0 + n / Gh of k sits k - 1 - q0 -
  // n / Gh before the end)
  const int hmax = p.k - 1 - p.q0;  // hidden positions of column 0, the most of any column
  int hid[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int n = 8 * nt + 2 * qd + c;
      hid[nt][c] = (n < G) ? p.k - 1 - p.q0 - n / p.Gh : 0;
    }
  uint64_t* wbar = bars + warp * NS;
  uint8_t* wtile = tiles + warp * NS * Gm::kTile;
  uint8_t* wside = sides + warp * NS * Gm::kSideStride;
  uint16_t* wq = qcopy + warp * NC * Gm::kQStride;
  float* woext = oext_all + warp * NC * Gm::kOStride;  // FP4: O of outlier channels [NC rows][D (+pad)]
  if constexpr (Gm::kFp4)
    for (int i = lane; i < NC * Gm::kOStride; i += 32) woext[i] = 0.f;
  const LdsmOffsets<KVF, D> lofs(lane);

  if (lane == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&wbar[s], 1);
    fence_mbar_init();
  }
  if (tid == 0) prefetch_tensormap(&tmap);

  // ---- prefix sums of blocks per sequence: P[b] = sum of ceil(L/16) below b ----
  {
    const int nthr = blockDim.x;
    const int per = (B + nthr - 1) / nthr;
    const int lo = min(B, tid * per), hi = min(B, lo + per);
    const int lim = kBlock * p.maxblk;
    int local = 0;
    for (int i = lo; i < hi; ++i) {
      const int L = p.seq_lens[i];
      const bool bad = (L < 0 || L > lim || (L > 0 && L < p.k));
      if (bad && blockIdx.x == 0) raise_flag(p.err, PQKV_DEVERR_SEQ_LEN);
      local += bad ? 0 : (L + kBlock - 1) / kBlock;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < warp; ++w) run += warp_sums[w];
    if (tid == 0) P[0] = 0;
    for (int i = lo; i < hi; ++i) {
      const int L = p.seq_lens[i];
      const bool bad = (L < 0 || L > lim || (L > 0 && L < p.k));
      run += bad ? 0 : (L + kBlock - 1) / kBlock;
      P[i + 1] = run;
    }
  }
  __syncthreads();

  // ---- sequences without blocks (empty or rejected): zero output rows ----
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (P[b + 1] != P[b]) continue;
    for (int i = tid; i < p.k * Hq * D; i += blockDim.x) store_out<QBF16>(p.out, (size_t)b * p.k * Hq * D + i, 0.f);
  }

  const int T = Hkv * P[B];
  const int W = gridDim.x * NW;
  const SplitPlan plan = make_split_plan(T, W, p.split_blocks);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  uint32_t phase = 0;     // parity bit per stage
  uint32_t inflight = 0;  // stages with an issued, unconsumed copy
  bool aborted = false;

  // flat block index -> (b, h, j) of its (sequence, head, block)
  auto locate = [&](int f, int& b, int& h, int& j) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (Hkv * P[mid] <= f) lo = mid; else hi = mid;
    }
    const int n = P[lo + 1] - P[lo];
    const int rel = f - Hkv * P[lo];
    b = lo;
    h = rel / n;
    j = rel - h * n;
  };

  // This warp's share of the flat range (see SplitPlan), cut into units at the
  // multiples of C inside it. Its blocks are numbered v = 0 .. Vtot - 1 from
  // f0w; the copy ring runs over v without a break at unit boundaries, and a
  // warp's units are mostly pieces of one (sequence, head) pair, so its query
  // stays loaded from one unit to the next.
  const int wr = warp * gridDim.x + blockIdx.x;
  const int f0w = (int)min((long long)T, (long long)wr * plan.Qw);
  const int f1w = min(T, f0w + plan.Qw);
  const int Vtot = f1w - f0w;
  auto vflat = [&](int v) { return f0w + v; };  // virtual block index -> flat block index
  // Per-lane window of (physical id, head) for blocks wbase + lane and, loaded
  // ahead, wbase + 32 + lane. Values are only inspected when issued.
  auto load_entry = [&](int v, int& id, int& hh) {
    id = -1;
    hh = 0;
    if (v < Vtot) {
      int b, h, j;
      locate(vflat(v), b, h, j);
      id = __ldg(p.block_tables + (size_t)b * p.maxblk + j);
      hh = h;
    }
  };
  int wbase = 0, wid, wh, nid, nh;
  load_entry(lane, wid, wh);
  load_entry(32 + lane, nid, nh);
  uint32_t skip = 0;
  // KV tiles are read once: evicted first, so that split partials stay in L2
  // until they are merged
  const uint64_t kv_policy = l2_evict_first_policy();
  auto issue = [&](int s, int v) {
    while (v - wbase >= 32) {
      wbase += 32;
      wid = nid;
      wh = nh;
      load_entry(wbase + 32 + lane, nid, nh);
    }
    const int id = __shfl_sync(kFull, wid, v - wbase);
    const int hh = __shfl_sync(kFull, wh, v - wbase);
    const bool bad = (id < 0 || id >= p.nb);
    inflight |= 1u << s;
    if (bad) skip |= 1u << s; else skip &= ~(1u << s);
    if (lane == 0) {
      uint64_t* bar = &wbar[s];
      if (bad) {
        raise_flag(p.err, PQKV_DEVERR_BLOCK_ID);
        mbar_arrive(bar);
      } else {
        const int coord = (id * Hkv + hh) * 32;
        mbar_arrive_expect_tx(bar, Gm::kTx);
        uint8_t* dst = wtile + s * Gm::kTile;
        constexpr int kElem = Gm::k16 ? 2 : 1;
#pragma unroll
        for (int bx = 0; bx < Gm::kBoxes; ++bx)
          tma_load_2d_hint(dst + bx * 32 * Gm::kBoxRow, &tmap, bx * (Gm::kBoxRow / kElem), coord, bar, kv_policy);
        const size_t pair = (size_t)id * Hkv + hh;
        uint8_t* side = wside + s * Gm::kSideStride;
        if constexpr (Gm::kFp8) {
          bulk_load(side, p.scales + pair * 16, 16, bar);
        } else if constexpr (Gm::kFp4) {
          bulk_load(side, p.scales + pair * Gm::kScaleBytes, Gm::kScaleBytes, bar);
          bulk_load(side + Gm::kScaleBytes, p.oval + pair * Gm::kValBytes, Gm::kValBytes, bar);
          bulk_load(side + Gm::kScaleBytes + Gm::kValBytes, p.oidx + pair * 16, 16, bar);
        }
      }
    }
  };
  for (int i = 0; i < min(NS, Vtot); ++i) issue(i, i);
  int s = 0;  // stage of the next block to consume

  // ---- consumer state of the current (sequence, head) piece ----
  int b = 0, h = 0, j = 0;
  int nblk = 0, Lb = 0;
  bool started_before = false;
  uint32_t qf[NT][KT][2];
  float acc[NT][KT][4];
  float mm[NT][2], ll[NT][2], vref;  // running max and sum of each of the lane's columns
  float rvref = 0.f;                  // FP8: 1 / vref (0 while vref is 0)
  // softmax scale (log2 units) of each of the lane's columns, times the power
  // of two its query row was scaled down by before narrowing to f16
  // (quantized caches; 16-bit caches keep the query in its own type)
  float csc[NT][2];
  OutlierState<NT> ost;  // FP4 only
  int qb = -1, qh = -1;  // the pair whose query is loaded
  int owed_k0 = -1, owed_n = 0;  // pieces of a long pair written but not yet published

  const int vb = -f0w;  // v = f + vb
  for (int f0 = f0w, f1 = f0w; f0 < f1w && !aborted; f0 = f1) {
    f1 = min(f1w, (f0 / plan.C + 1) * plan.C);  // this unit: [f0, f1)
    const int k = plan.unit(f0);

    locate(f0, b, h, j);
    nblk = P[b + 1] - P[b];
    Lb = p.seq_lens[b];
    started_before = j > 0;

    // a new piece: zero the softmax state; load the pair's query unless the
    // previous piece of this warp was of the same pair
    auto begin_piece = [&]() {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mm[nt][0] = mm[nt][1] = kNegInf;
        ll[nt][0] = ll[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < KT; ++mt) acc[nt][mt][0] = acc[nt][mt][1] = acc[nt][mt][2] = acc[nt][mt][3] = 0.f;
      }
      vref = 0.f;
      rvref = 0.f;
      if (b == qb && h == qh) return;
      qb = b;
      qh = h;
      ost.reset();  // the query changes
      float rowmul[NT];  // quantized caches: 2^-e applied to this lane's query row 8nt + g
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
      const bool has = 8 * nt + g < G;
      const size_t qrow = has ? col_row(b, h, 8 * nt + g, p.k, p.q0, p.Gh, Hq, D) : 0;
      // k-slot order of the dequantized K fragments: FP8 k-step kk holds
      // d = 16kk + 4qd + {0,1 | 2,3}; FP4 k-step (c, s) = (kk/2, kk%2) holds
      // d = 32c + 8qd + 4s + {0,1 | 2,3}.
      auto d0_of = [&](int kk) { return Gm::kFp8 ? 16 * kk + 4 * qd : 32 * (kk >> 1) + 8 * qd + 4 * (kk & 1); };
      rowmul[nt] = 1.f;
      if constexpr (!Gm::k16 && QBF16) {
        // A bf16 row is narrowed to f16 for the MMA: scale it by the power of two
        // 2^-e that brings its largest |q| into [2^13, 2^14) (exact, and far
        // from both ends of the f16 range); the logits of its column are
        // multiplied back by 2^e in the softmax.
        float mx = 0.f;
        if (has) {
#pragma unroll
          for (int kk = 0; kk < KT; ++kk)
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fabsf(q_at<QBF16>(p.q, qrow + d0_of(kk) + i)));
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const int ex = (mx > 0.f && mx <= FLT_MAX) ? ilogbf(mx) - 13 : 0;
        rowmul[nt] = ldexpf(1.f, -ex);
      }
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        if constexpr (Gm::k16) {
          const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
          qf[nt][kk][0] = has ? __ldg(q32 + (qrow + 16 * kk + 2 * qd) / 2) : 0u;
          qf[nt][kk][1] = has ? __ldg(q32 + (qrow + 16 * kk + 8 + 2 * qd) / 2) : 0u;
        } else {
          const int d0 = d0_of(kk);
          float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
          if (has) {
            v0 = q_at<QBF16>(p.q, qrow + d0) * rowmul[nt];
            v1 = q_at<QBF16>(p.q, qrow + d0 + 1) * rowmul[nt];
            v2 = q_at<QBF16>(p.q, qrow + d0 + 2) * rowmul[nt];
            v3 = q_at<QBF16>(p.q, qrow + d0 + 3) * rowmul[nt];
          }
          qf[nt][kk][0] = f16x2_from(v0, v1);
          qf[nt][kk][1] = f16x2_from(v2, v3);
        }
      }
      // column c of this lane is query row 2qd + c of the tile, held by lanes g = 2qd + c
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float m = __shfl_sync(kFull, rowmul[nt], (2 * qd + c) << 2);
        csc[nt][c] = (Gm::k16 || !QBF16) ? p.scale_log2 : p.scale_log2 / m;  // 1 / m = 2^e: exact
      }
      }
      if constexpr (Gm::kFp4) {
        // f16 copy of this warp's query rows for the outlier channels, scaled
        // like the fragments (the row of element i is the same on all lanes)
        __syncwarp();
        for (int i = lane; i < NC * D; i += 32) {
          const int n = i / D;
          const float m = __shfl_sync(kFull, rowmul[n >> 3 < NT ? n >> 3 : 0], (n & 7) << 2);
          const float v = (n < G) ? q_at<QBF16>(p.q, col_row(b, h, n, p.k, p.q0, p.Gh, Hq, D) + (i % D)) * m : 0.f;
          wq[n * Gm::kQStride + i % D] = __half_as_ushort(__float2half_rn(v));
        }
        __syncwarp();
      }
    };

    auto finish_piece = [&](bool ends_after) {
      float lt[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        lt[nt][0] = ll[nt][0];
        lt[nt][1] = ll[nt][1];
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          lt[nt][0] += __shfl_xor_sync(kFull, lt[nt][0], o);
          lt[nt][1] += __shfl_xor_sync(kFull, lt[nt][1], o);
        }
      }
      const float vs = Gm::kFp8 ? vref : 1.f;
      if constexpr (Gm::kFp4) {  // fold the outlier channels' O in and clear it
        ost.template flush<Gm::kOStride>(woext, lane, D);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < KT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float* slot = woext + (8 * nt + 2 * qd + (e & 1)) * Gm::kOStride + dmap<KVF>(mt, g + 8 * (e >> 1));
              acc[nt][mt][e] += *slot;
              *slot = 0.f;
            }
        __syncwarp();
      }
      if (!started_before && !ends_after) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int n0 = 8 * nt + 2 * qd, n1 = n0 + 1;
          const float i0 = lt[nt][0] > 0.f ? vs / lt[nt][0] : 0.f;
          const float i1 = lt[nt][1] > 0.f ? vs / lt[nt][1] : 0.f;
          const size_t ob0 = n0 < G ? col_row(b, h, n0, p.k, p.q0, p.Gh, Hq, D) : 0;
          const size_t ob1 = n1 < G ? col_row(b, h, n1, p.k, p.q0, p.Gh, Hq, D) : 0;
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            const int da = dmap<KVF>(mt, g), db = dmap<KVF>(mt, g + 8);
            if constexpr (!Gm::k16) {  // rows g, g + 8 of an m-tile are head dims da, da + 1: one 4-byte store
              if (n0 < G) store_out2<QBF16>(p.out, ob0 + da, acc[nt][mt][0] * i0, acc[nt][mt][2] * i0);
              if (n1 < G) store_out2<QBF16>(p.out, ob1 + da, acc[nt][mt][1] * i1, acc[nt][mt][3] * i1);
            } else {
              if (n0 < G) {
                store_out<QBF16>(p.out, ob0 + da, acc[nt][mt][0] * i0);
                store_out<QBF16>(p.out, ob0 + db, acc[nt][mt][2] * i0);
              }
              if (n1 < G) {
                store_out<QBF16>(p.out, ob1 + da, acc[nt][mt][1] * i1);
                store_out<QBF16>(p.out, ob1 + db, acc[nt][mt][3] * i1);
              }
            }
          }
        }
        return;
      }
      const int slot = started_before ? 2 * k : 2 * k + 1;
      float* base = p.partials + (size_t)slot * p.slot_floats;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n0 = 8 * nt + 2 * qd, n1 = n0 + 1;
#pragma unroll
        for (int mt = 0; mt < KT; ++mt) {
          const int da = dmap<KVF>(mt, g), db = dmap<KVF>(mt, g + 8);
          if constexpr (!Gm::k16) {  // head dims da, da + 1 (da even): one 8-byte store
            if (n0 < G)
              *reinterpret_cast<float2*>(base + n0 * D + da) = make_float2(acc[nt][mt][0] * vs, acc[nt][mt][2] * vs);
            if (n1 < G)
              *reinterpret_cast<float2*>(base + n1 * D + da) = make_float2(acc[nt][mt][1] * vs, acc[nt][mt][3] * vs);
          } else {
            if (n0 < G) {
              base[n0 * D + da] = acc[nt][mt][0] * vs;
              base[n0 * D + db] = acc[nt][mt][2] * vs;
            }
            if (n1 < G) {
              base[n1 * D + da] = acc[nt][mt][1] * vs;
              base[n1 * D + db] = acc[nt][mt][3] * vs;
            }
          }
        }
        if (g == 0) {
          if (n0 < G) {
            base[G * D + n0] = mm[nt][0];
            base[G * D + G + n0] = lt[nt][0];
          }
          if (n1 < G) {
            base[G * D + n1] = mm[nt][1];
            base[G * D + G + n1] = lt[nt][1];
          }
        }
      }
      // every piece is counted in its pair's arrival word. A pair of at most
      // kMergeInKernel pieces is merged at once by the warp that brings its
      // last piece. A longer one is merged column by column after the warps'
      // shares, so its pieces are only counted here and published together
      // when the warp moves on to another pair (one fence for all of them).
      __syncwarp();
      const int s0 = Hkv * P[b] + h * nblk;  // flat index of the pair's first block
      const int k0 = plan.unit(s0), np = plan.unit(s0 + nblk - 1) - k0 + 1;
      if (np <= kMergeInKernel) {
        if (arrive_split(p, k0, np, lane)) merge_pair<D, QBF16>(p, b, h, k0, np, lane);
      } else {
        if (k0 != owed_k0) {
          publish_pieces(p, owed_k0, owed_n, lane);
          owed_n = 0;
        }
        owed_k0 = k0;
        ++owed_n;
      }
    };

    // A stage whose wait gives up keeps its phase and its in-flight bit, so
    // that the drain below waits for that very copy.
    auto wait_stage = [&](int s) -> bool {
      const bool ok = __all_sync(kFull, mbar_wait_bounded(&wbar[s], (phase >> s) & 1u, p.timeout_ns));
      if (ok) {
        phase ^= 1u << s;
        inflight &= ~(1u << s);
      }
      return ok;
    };

    begin_piece();
    int f = f0;
    while (f < f1) {
      // two consecutive blocks of the same piece when available, else one
      const int n2 = (f + 1 < f1 && j + 1 < nblk) ? 2 : 1;
      const int sA = s, sB = (s + 1 == NS) ? 0 : s + 1;
      bool ok = wait_stage(sA);
      if (n2 == 2) ok = wait_stage(sB) && ok;
      if (!ok) {
        if (lane == 0) raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
        aborted = true;
        break;
      }
      const bool useA = !((skip >> sA) & 1u);
      const bool useB = (n2 == 2) && !((skip >> sB) & 1u);
      const int remA = Lb - kBlock * j, remB = remA - kBlock;  // tokens left from each block on
      const int validA = min(kBlock, remA), validB = min(kBlock, remB);
      const uint32_t tbA = smem_u32(wtile + sA * Gm::kTile), tbB = smem_u32(wtile + sB * Gm::kTile);
      const uint8_t* sdA = wside + sA * Gm::kSideStride;
      const uint8_t* sdB = wside + sB * Gm::kSideStride;

      // ---- scores of both blocks (independent MMA chains) ----
      float scA[NT][4], scB[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) scA[nt][e] = scB[nt][e] = 0.f;
      if (useA) block_scores<KVF, D, NT>(tbA, sdA, qf, wq, lofs, lane, scA, ost);
      if (useB) block_scores<KVF, D, NT>(tbB, sdB, qf, wq, lofs, lane, scB, ost);
      float skA = 1.f, skB = 1.f, svA = 1.f, svB = 1.f;
      if constexpr (Gm::kFp8) {
        if (useA) { skA = reinterpret_cast<const float*>(sdA)[0]; svA = reinterpret_cast<const float*>(sdA)[1]; }
        if (useB) { skB = reinterpret_cast<const float*>(sdB)[0]; svB = reinterpret_cast<const float*>(sdB)[1]; }
      }

      // ---- online softmax over up to 32 tokens (log2 domain) ----
      // x[nt][e]: row (token) g + 8 (e >> 1), column 8nt + 2qd + (e & 1)
      float xA[NT][4], xB[NT][4], bm[NT][2];
      bool need_any = false;
      constexpr float kLazy = lazy_of<KVF>();
      // both blocks full and visible to every column (the usual case): no mask
      const bool full2 = useA && useB && remB - hmax >= kBlock;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float mA0 = csc[nt][0] * skA, mA1 = csc[nt][1] * skA;
        const float mB0 = csc[nt][0] * skB, mB1 = csc[nt][1] * skB;
        if (full2) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xA[nt][e] = scA[nt][e] * ((e & 1) ? mA1 : mA0);
            xB[nt][e] = scB[nt][e] * ((e & 1) ? mB1 : mB0);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = g + 8 * (e >> 1), hd = hid[nt][e & 1];
            // column n sees the tokens before the last hid ones (0 for one query token)
            xA[nt][e] = (!useA || r >= remA - hd) ? kNegInf : scA[nt][e] * ((e & 1) ? mA1 : mA0);
            xB[nt][e] = (!useB || r >= remB - hd) ? kNegInf : scB[nt][e] * ((e & 1) ? mB1 : mB0);
          }
        }
        bm[nt][0] = fmaxf(fmaxf(xA[nt][0], xA[nt][2]), fmaxf(xB[nt][0], xB[nt][2]));
        bm[nt][1] = fmaxf(fmaxf(xA[nt][1], xA[nt][3]), fmaxf(xB[nt][1], xB[nt][3]));
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          bm[nt][0] = fmaxf(bm[nt][0], __shfl_xor_sync(kFull, bm[nt][0], o));
          bm[nt][1] = fmaxf(bm[nt][1], __shfl_xor_sync(kFull, bm[nt][1], o));
        }
        need_any |= (bm[nt][0] > mm[nt][0] + kLazy) || (bm[nt][1] > mm[nt][1] + kLazy);
      }
      float fc[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) fc[nt][0] = fc[nt][1] = 1.f;
      bool rescale = __any_sync(kFull, need_any);
      if (rescale) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (bm[nt][c] > mm[nt][c] + kLazy) {
              fc[nt][c] = ex2(mm[nt][c] - bm[nt][c]);
              mm[nt][c] = bm[nt][c];
            }
            ll[nt][c] *= fc[nt][c];
          }
      }
      // FP8 V scales: O is kept in units of vref, the largest V scale so far;
      // a block with a smaller scale enters with P scaled by sv / vref <= 1.
      float prA = 1.f, prB = 1.f;
      if constexpr (Gm::kFp8) {
        const float svm = fmaxf(useA ? svA : 0.f, useB ? svB : 0.f);
        if (svm > vref) {
          const float rs = vref / svm;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            fc[nt][0] *= rs;
            fc[nt][1] *= rs;
          }
          vref = svm;
          rvref = 1.f / svm;  // only when the largest scale grows
          rescale = true;
        }
        prA = useA ? svA * rvref : 0.f;  // <= 1; differs from svA / vref by an ulp at most
        prB = useB ? svB * rvref : 0.f;
      }
      if (rescale) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            acc[nt][mt][0] *= fc[nt][0];
            acc[nt][mt][1] *= fc[nt][1];
            acc[nt][mt][2] *= fc[nt][0];
            acc[nt][mt][3] *= fc[nt][1];
          }
        if constexpr (Gm::kFp4) {  // the outlier channels' O follows the same rescale
          __syncwarp();
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            ost.vacc[nt][0] *= fc[nt][0];
            ost.vacc[nt][1] *= fc[nt][1];
#pragma unroll
            for (int mt = 0; mt < KT; ++mt)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                woext[(8 * nt + 2 * qd + (e & 1)) * Gm::kOStride + dmap<KVF>(mt, g + 8 * (e >> 1))] *=
                    fc[nt][e & 1];
          }
          __syncwarp();
        }
      }
      float pA[NT][4], pB[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mc = mm[nt][e & 1];
          const bool live = mc != kNegInf;
          pA[nt][e] = live ? ex2(xA[nt][e] - mc) : 0.f;
          pB[nt][e] = live ? ex2(xB[nt][e] - mc) : 0.f;
        }
        ll[nt][0] += (pA[nt][0] + pA[nt][2]) + (pB[nt][0] + pB[nt][2]);
        ll[nt][1] += (pA[nt][1] + pA[nt][3]) + (pB[nt][1] + pB[nt][3]);
      }

      // ---- O^T += V^T P^T; P = P_hi + P_lo (except FP4) so ~16 significant bits survive ----
      auto pv = [&](uint32_t tb, const uint8_t* sd, int valid, const float (&w)[NT][4], float pr) {
        uint32_t b0[NT], b1[NT], c0[NT], c1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float w0 = w[nt][0] * pr, w1 = w[nt][1] * pr, w2 = w[nt][2] * pr, w3 = w[nt][3] * pr;
          const uint32_t hA = pack_f32x2(w0, w1, kBf16Mma), hB = pack_f32x2(w2, w3, kBf16Mma);
          b0[nt] = movmatrix_t(hA);
          b1[nt] = movmatrix_t(hB);
          if constexpr (Gm::kFp4) {
            c0[nt] = c1[nt] = 0u;
          } else {
            const uint32_t lA = pack_f32x2(w0 - unpack_lo(hA, kBf16Mma), w1 - unpack_hi(hA, kBf16Mma), kBf16Mma);
            const uint32_t lB = pack_f32x2(w2 - unpack_lo(hB, kBf16Mma), w3 - unpack_hi(hB, kBf16Mma), kBf16Mma);
            c0[nt] = movmatrix_t(lA);
            c1[nt] = movmatrix_t(lB);
          }
        }
        block_pv<KVF, D, NT>(tb, sd, lofs, lane, valid, b0, b1, c0, c1, acc, woext, ost);
      };
      if (useA && (!Gm::kFp8 || prA > 0.f)) pv(tbA, sdA, validA, pA, prA);
      if (useB && (!Gm::kFp8 || prB > 0.f)) pv(tbB, sdB, validB, pB, prB);

      __syncwarp();
      const int v = f + vb;
      if (v + NS < Vtot) issue(sA, v + NS);
      if (n2 == 2 && v + 1 + NS < Vtot) issue(sB, v + 1 + NS);
      s = (sB + 1 == NS) ? 0 : sB + 1;
      if (n2 == 1) s = sB;

      // ---- advance through (sequence, head, block) ----
      f += n2;
      j += n2;
      const bool seg_end = (j == nblk);
      const bool chunk_end = (f == f1);
      if (seg_end || chunk_end) {
        finish_piece(!seg_end);
        if (!chunk_end) {
          j = 0;
          if (++h == Hkv) {
            h = 0;
            do { ++b; } while (P[b + 1] == P[b]);
            nblk = P[b + 1] - P[b];
            Lb = p.seq_lens[b];
          }
          started_before = false;
          begin_piece();
        }
      }
    }
  }

  publish_pieces(p, owed_k0, owed_n, lane);

  // ---- long split pairs (more than kMergeInKernel pieces): output column c
  // of all (sequence, head, query row) columns is merged by warp c mod W, once
  // its pair's pieces are all written ----
  if (!aborted) {
    const long ncols = (long)B * Hkv * G;
    for (long c = wr; c < ncols; c += W) {
      const int cb = (int)(c / ((long)Hkv * G));
      const int ch = (int)((c / G) % Hkv), cn = (int)(c % G);
      const int cnb = P[cb + 1] - P[cb];
      if (cnb == 0) continue;
      const int s0 = Hkv * P[cb] + ch * cnb;
      const int k0 = plan.unit(s0), np = plan.unit(s0 + cnb - 1) - k0 + 1;
      if (np <= kMergeInKernel) continue;
      if (!wait_pieces(p, k0, np, lane)) {
        if (lane == 0) raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
        continue;
      }
      // pieces loaded at once: as many as the registers the main loop leaves allow
      merge_column<D, QBF16, Gm::k16 ? 32 : 24>(p, cb, ch, cn, k0, np, lane);
    }
  }

  // after a timeout: let copies still in flight land before the warp exits
  // (with the full limit, whatever the limit that gave up)
  if (aborted) {
    bool drained = true;
    for (int s2 = 0; s2 < NS; ++s2)
      if ((inflight >> s2) & 1u) drained = mbar_wait_bounded(&wbar[s2], (phase >> s2) & 1u, p.drain_ns) && drained;
    if (!drained && lane == 0) raise_flag(p.err, PQKV_DEVERR_DRAIN);
  }
}

// ---- instantiation + launch --------------------------------------------------

template <int KVF, int D, bool QBF16, int NT>
static cudaError_t launch_decode_t(const CUtensorMap& tmap, const DecodeParams& p, int grid, cudaStream_t st) {
  auto kern = paged_decode_kernel<KVF, D, QBF16, NT>;
  const size_t smem = DecodeSmem<KVF, D, NT>::bytes(p.B);
  // opt in once per device to the largest size any batch can need
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)DecodeSmem<KVF, D, NT>::bytes(PQKV_MAX_BATCH));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  // programmatic dependent of whatever precedes it on the stream (usually the
  // cache write): the kernel waits for that grid before its first read, so
  // only the launch overlaps
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(DecodeGeom<KVF, D, NT>::kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmap, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// nt = tiles of 8 MMA columns per warp (1, or 2 for up to 16 query rows per KV head)
template <int NT>
static size_t decode_smem_bytes_t(int kv_dtype, int D, int B) {
  switch (kv_dtype) {
    case PQKV_DTYPE_FP16:
    case PQKV_DTYPE_BF16:
      return D == 128 ? DecodeSmem<PQKV_DTYPE_BF16, 128, NT>::bytes(B) : DecodeSmem<PQKV_DTYPE_BF16, 64, NT>::bytes(B);
    case PQKV_DTYPE_FP8_E4M3:
    case PQKV_DTYPE_FP8_E5M2:
      return D == 128 ? DecodeSmem<PQKV_DTYPE_FP8_E4M3, 128, NT>::bytes(B)
                      : DecodeSmem<PQKV_DTYPE_FP8_E4M3, 64, NT>::bytes(B);
    default:
      return D == 128 ? DecodeSmem<PQKV_DTYPE_FP4_E2M1, 128, NT>::bytes(B)
                      : DecodeSmem<PQKV_DTYPE_FP4_E2M1, 64, NT>::bytes(B);
  }
}

size_t decode_smem_bytes(int kv_dtype, int D, int B, int nt) {
  return nt == 2 ? decode_smem_bytes_t<2>(kv_dtype, D, B) : decode_smem_bytes_t<1>(kv_dtype, D, B);
}

cudaError_t launch_decode(int kv_dtype, int D, bool q_bf16, int nt, const CUtensorMap& tmap, const DecodeParams& p,
                          int grid, cudaStream_t st) {
#define PQKV_DEC(KVF, DD, QB)                                                                        \
  if (kv_dtype == KVF && D == DD && q_bf16 == QB)                                                    \
    return nt == 2 ? launch_decode_t<KVF, DD, QB, 2>(tmap, p, grid, st)                              \
                   : launch_decode_t<KVF, DD, QB, 1>(tmap, p, grid, st);
  PQKV_DEC(PQKV_DTYPE_FP16, 128, false)
  PQKV_DEC(PQKV_DTYPE_FP16, 64, false)
  PQKV_DEC(PQKV_DTYPE_BF16, 128, true)
  PQKV_DEC(PQKV_DTYPE_BF16, 64, true)
  PQKV_DEC(PQKV_DTYPE_FP8_E4M3, 128, true)
  PQKV_DEC(PQKV_DTYPE_FP8_E4M3, 128, false)
  PQKV_DEC(PQKV_DTYPE_FP8_E4M3, 64, true)
  PQKV_DEC(PQKV_DTYPE_FP8_E4M3, 64, false)
  PQKV_DEC(PQKV_DTYPE_FP8_E5M2, 128, true)
  PQKV_DEC(PQKV_DTYPE_FP8_E5M2, 128, false)
  PQKV_DEC(PQKV_DTYPE_FP8_E5M2, 64, true)
  PQKV_DEC(PQKV_DTYPE_FP8_E5M2, 64, false)
  PQKV_DEC(PQKV_DTYPE_FP4_E2M1, 128, true)
  PQKV_DEC(PQKV_DTYPE_FP4_E2M1, 128, false)
  PQKV_DEC(PQKV_DTYPE_FP4_E2M1, 64, true)
  PQKV_DEC(PQKV_DTYPE_FP4_E2M1, 64, false)
#undef PQKV_DEC
  return cudaErrorInvalidValue;
}

}  // namespace pqkv
