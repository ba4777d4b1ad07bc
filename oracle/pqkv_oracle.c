/*
 * pqkv_oracle.c -- TEST INFRASTRUCTURE ONLY: the CPU oracle.
 *
 * A plain, slow, obviously correct restatement of what the paged, quantized KV
 * cache computes, used to check the GPU library. Only the test suite, the
 * package smoke check and the benchmark's CPU-baseline leg may load it. It
 * shares no code, header, table or constant with the GPU library.
 *
 * Sources (cited by page title and section):
 *  [P1] "vLLM 0.7 Ships Unified KV Cache Compression" -- "Technical Breakdown:
 *       Dynamic Quantization with Outlier Retention", steps 1-4; architecture
 *       diagram (FP16 outlier buffer, Flash-Decoding kernel).
 *  [P2] "vLLM v0.7.2" field report -- "Deconstructing the v0.7.2 Architecture"
 *       (FP8 E4M3/E5M2 KV cache, 16-token blocks, page tables).
 *  [P3] "vLLM" glossary -- "PagedAttention" (logical-to-physical block mapping,
 *       blocks shared across sequences), "KV cache quantization", "Chunked
 *       prefill" (long prompts processed in chunks).
 *  [OFP8] OCP 8-bit Floating Point Specification: E4M3 (bias 7, max 448, no
 *       infinities, S.1111.111 = NaN) and E5M2 (bias 15, max 57344, IEEE-like).
 *  [MX] OCP Microscaling Formats specification: E2M1 (bias 1, values
 *       0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities or NaN).
 * Readings where the pages are silent (scale granularity, the statistic behind
 * "3.2 sigma", outlier capacity, FP8 append) are stated at each function.
 *
 * Floating point: fp64 for attention; the quantizer's own steps in fp32 exactly
 * as stated (IEEE division, round to nearest even); the outlier statistics in
 * fp64 in channel order. Build with -ffp-contract=off so that no multiply-add
 * is fused.
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { DT_FP16 = 0, DT_BF16 = 1, DT_E4M3 = 2, DT_E5M2 = 3, DT_E2M1 = 4 };
enum { ERR_SLOT = 1, ERR_BLOCK_ID = 2, ERR_SEQ_LEN = 4, ERR_RUN = 8 };
enum { BS = 16, R_OUT = 4, IDX_STRIDE = 8, GROUP = 16 };

/* ------------------------------------------------------------------------ */
/* Small floating-point formats, from their definitions ([OFP8], [MX], IEEE).  */
/* ------------------------------------------------------------------------ */

typedef struct {
  int ebits, mbits, bias;
  int max_code;      /* largest finite magnitude code */
  int ieee_overflow; /* 1: overflow goes to infinity (IEEE binary16) */
} minifloat;

static const minifloat F_E4M3 = {4, 3, 7, 0x7E, 0};
static const minifloat F_E5M2 = {5, 2, 15, 0x7B, 0};
static const minifloat F_E2M1 = {2, 1, 1, 0x7, 0};
static const minifloat F_FP16 = {5, 10, 15, 0x7BFF, 1};

static const minifloat* fmt_of(int dt) {
  switch (dt) {
    case DT_E4M3: return &F_E4M3;
    case DT_E5M2: return &F_E5M2;
    case DT_E2M1: return &F_E2M1;
    case DT_FP16: return &F_FP16;
    default: return 0;
  }
}

/* Value of a code: sign, biased exponent field e, mantissa field m.
 * e == 0: m * 2^(1 - bias - mbits) (subnormal); else (2^mbits + m) *
 * 2^(e - bias - mbits). E4M3 has no infinity and only S.1111.111 is NaN;
 * E5M2 and binary16 reserve the all-ones exponent for inf/NaN. */
static double mf_decode(const minifloat* f, uint32_t code) {
  uint32_t sign = (code >> (f->ebits + f->mbits)) & 1u;
  uint32_t e = (code >> f->mbits) & ((1u << f->ebits) - 1u);
  uint32_t m = code & ((1u << f->mbits) - 1u);
  uint32_t emax = (1u << f->ebits) - 1u;
  double mag;
  if (f == &F_E4M3 && e == emax && m == (1u << f->mbits) - 1u) return NAN;
  if ((f == &F_E5M2 || f == &F_FP16) && e == emax) {
    mag = (m == 0) ? INFINITY : NAN;
    return sign ? -mag : mag;
  }
  if (e == 0)
    mag = ldexp((double)m, 1 - f->bias - f->mbits);
  else
    mag = ldexp((double)((1u << f->mbits) + m), (int)e - f->bias - f->mbits);
  return sign ? -mag : mag;
}

/* Round a finite float to the nearest value of the format, ties to the even
 * code, keeping the sign (also of zero). Magnitudes past the largest finite
 * value saturate to it ("satfinite"), except for IEEE binary16 where they
 * round to infinity. Works on the exact binary expansion of x: with
 * x = M * 2^(E-23), M the 24-bit significand, the result is the integer
 * r = round(x / 2^(e_eff - mbits)), e_eff = max(E, emin), emin = 1 - bias,
 * and the code is ((e_eff + bias - 1) << mbits) + r, which carries into the
 * exponent field exactly when r reaches the next binade. */
static uint32_t mf_encode(const minifloat* f, float x) {
  uint32_t u;
  memcpy(&u, &x, sizeof u);
  uint32_t sbit = (u >> 31) << (f->ebits + f->mbits);
  uint32_t a = u & 0x7FFFFFFFu;
  if (a >= 0x7F800000u) /* infinities (NaN is outside the domain) */
    return sbit | (f->ieee_overflow ? (uint32_t)(f->max_code + 1) : (uint32_t)f->max_code);
  if ((a >> 23) == 0) /* zero or fp32 subnormal: below half of every quantum */
    return sbit;
  int E = (int)(a >> 23) - 127;
  uint64_t M = (a & 0x7FFFFFu) | 0x800000u;
  int emin = 1 - f->bias;
  int eeff = E > emin ? E : emin;
  int shift = 23 - f->mbits + (eeff - E); /* low bits of M below the quantum */
  uint64_t r;
  if (shift > 24) {
    r = 0;
  } else {
    uint64_t rem = M & ((1ull << shift) - 1ull);
    uint64_t half = 1ull << (shift - 1);
    r = M >> shift;
    if (rem > half || (rem == half && (r & 1ull))) r += 1;
  }
  int64_t code = ((int64_t)(eeff + f->bias - 1) << f->mbits) + (int64_t)r;
  if (f->ieee_overflow) {
    if (code > f->max_code) code = f->max_code + 1; /* infinity */
  } else if (code > f->max_code) {
    code = f->max_code;
  }
  return sbit | (uint32_t)code;
}

static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Exported format helpers (for the oracle's own pins). */
void oracle_encode(int dt, const float* x, int64_t n, uint8_t* out) {
  const minifloat* f = fmt_of(dt);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)mf_encode(f, x[i]);
}

void oracle_encode_fp16(const float* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint16_t)mf_encode(&F_FP16, x[i]);
}

void oracle_decode(int dt, const uint8_t* codes, int64_t n, double* out) {
  const minifloat* f = fmt_of(dt);
  for (int64_t i = 0; i < n; ++i) out[i] = mf_decode(f, codes[i]);
}

void oracle_decode_fp16(const uint16_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = mf_decode(&F_FP16, codes[i]);
}

/* ------------------------------------------------------------------------ */
/* Cache geometry: one (block, head) pair = K tile then V tile, 16 tokens.     */
/* ------------------------------------------------------------------------ */

typedef struct {
  int dt, nb, H, D;
  uint8_t* cache;   /* [nb][H][2][16][row] */
  uint8_t* scales;  /* FP8: float [nb][H][4]; FP4: u8 [nb][H][2][16][D/16] */
  uint8_t* oidx;    /* FP4: u8 [nb][H][2][8] */
  uint8_t* oval;    /* FP4: fp16 [nb][H][2][16][4] */
} cache_t;

static size_t row_bytes(const cache_t* c) {
  if (c->dt == DT_FP16 || c->dt == DT_BF16) return (size_t)c->D * 2;
  if (c->dt == DT_E2M1) return (size_t)c->D / 2;
  return (size_t)c->D;
}

/* index of (block, head, kv) tile */
static size_t tile_index(const cache_t* c, int blk, int h, int kv) {
  return ((size_t)blk * c->H + h) * 2 + kv;
}

static uint8_t* row_ptr(const cache_t* c, int blk, int h, int kv, int t) {
  return c->cache + (tile_index(c, blk, h, kv) * BS + t) * row_bytes(c);
}

static float* fp8_scale_ptr(const cache_t* c, int blk, int h, int kv) {
  return (float*)(c->scales + (((size_t)blk * c->H + h) * 4 + kv) * sizeof(float));
}

static uint8_t* fp4_scale_ptr(const cache_t* c, int blk, int h, int kv, int t) {
  return c->scales + (tile_index(c, blk, h, kv) * BS + t) * (size_t)(c->D / GROUP);
}

static uint8_t* fp4_idx_ptr(const cache_t* c, int blk, int h, int kv) {
  return c->oidx + tile_index(c, blk, h, kv) * IDX_STRIDE;
}

static uint16_t* fp4_val_ptr(const cache_t* c, int blk, int h, int kv, int t) {
  return (uint16_t*)(c->oval + ((tile_index(c, blk, h, kv) * BS + t) * R_OUT) * 2);
}

/* Where the E2M1 code of (token t, channel ch) lives, and in which nibble.
 * The storage order is this library's own (the pages fix none):
 *  K tile: row t holds token t; byte i = channels 2i (low nibble), 2i + 1.
 *  V tile: byte = one channel of two tokens. Tokens (t, t + 1), t even, form a
 *    pair; pair p = 2k (k < 4) is tokens (2k, 2k + 1), pair 2k + 1 is tokens
 *    (2k + 8, 2k + 9); the even token is the low nibble. Channels [0, D/2) of
 *    pair p sit in row p, channels [D/2, D) in row 8 + p, byte = ch mod D/2. */
static uint8_t* fp4_code_byte(const cache_t* c, int blk, int h, int kv, int t, int ch, int* shift) {
  if (kv == 0) {
    *shift = (ch & 1) ? 4 : 0;
    return row_ptr(c, blk, h, kv, t) + ch / 2;
  }
  const int half = c->D / 2;
  const int pair = (t < 8) ? (t & ~1) : (((t - 8) & ~1) + 1);
  *shift = (t & 1) ? 4 : 0;
  return row_ptr(c, blk, h, kv, (ch / half) * 8 + pair) + ch % half;
}

static int fp4_get_code(const cache_t* c, int blk, int h, int kv, int t, int ch) {
  int shift;
  const uint8_t byte = *fp4_code_byte(c, blk, h, kv, t, ch, &shift);
  return (byte >> shift) & 0xF;
}

static void fp4_set_code(const cache_t* c, int blk, int h, int kv, int t, int ch, int code) {
  int shift;
  uint8_t* p = fp4_code_byte(c, blk, h, kv, t, ch, &shift);
  *p = (uint8_t)((*p & ~(0xF << shift)) | (code << shift));
}

/* Dequantized value of channel ch of token offset t ([P1] step 4 for FP4: the
 * outlier buffer's fp16 value where the channel is an outlier, else
 * e2m1(code) * e4m3(group scale); FP8: decode(code) * block scale). */
static double dequant(const cache_t* c, int blk, int h, int kv, int t, int ch) {
  switch (c->dt) {
    case DT_FP16: {
      uint16_t b;
      memcpy(&b, row_ptr(c, blk, h, kv, t) + (size_t)ch * 2, 2);
      return mf_decode(&F_FP16, b);
    }
    case DT_BF16: {
      uint16_t b;
      memcpy(&b, row_ptr(c, blk, h, kv, t) + (size_t)ch * 2, 2);
      return (double)bf16_to_f32(b);
    }
    case DT_E4M3:
    case DT_E5M2: {
      const minifloat* f = fmt_of(c->dt);
      double s = (double)*fp8_scale_ptr(c, blk, h, kv);
      return mf_decode(f, row_ptr(c, blk, h, kv, t)[ch]) * s;
    }
    default: {
      const uint8_t* idx = fp4_idx_ptr(c, blk, h, kv);
      for (int r = 0; r < R_OUT; ++r)
        if (idx[r] < c->D && idx[r] == ch) return mf_decode(&F_FP16, fp4_val_ptr(c, blk, h, kv, t)[r]);
      double sc = mf_decode(&F_E4M3, fp4_scale_ptr(c, blk, h, kv, t)[ch / GROUP]);
      return mf_decode(&F_E2M1, (uint32_t)fp4_get_code(c, blk, h, kv, t, ch)) * sc;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Cache write                                                                */
/* ------------------------------------------------------------------------ */

static float in_value(const uint16_t* x, int in_dt, size_t idx) {
  if (in_dt == DT_BF16) return bf16_to_f32(x[idx]);
  return (float)mf_decode(&F_FP16, x[idx]);
}

/* FP8 write of one run ([P2] FP8 E4M3/E5M2 KV cache; [P3] just-in-time
 * quantization). Reading: one fp32 absmax scale per (block, KV head, K|V);
 * a run starting at offset 0 opens the block; a later run may only grow the
 * scale, re-encoding the codes already in the block. */
static void write_fp8_run(const cache_t* c, const uint16_t* x, int in_dt, int t0, int n,
                          int blk, int off0, int h, int kv) {
  const minifloat* f = fmt_of(c->dt);
  const float fpmax = (c->dt == DT_E4M3) ? 448.0f : 57344.0f;
  const size_t tok_stride = (size_t)c->H * c->D;
  float a = 0.0f;
  for (int j = 0; j < n; ++j)
    for (int ch = 0; ch < c->D; ++ch) {
      float v = fabsf(in_value(x, in_dt, (size_t)(t0 + j) * tok_stride + (size_t)h * c->D + ch));
      if (v > a) a = v;
    }
  float s_run = a / fpmax;
  float* sp = fp8_scale_ptr(c, blk, h, kv);
  float s;
  if (off0 == 0) {
    s = s_run;
  } else {
    float s_old = *sp;
    s = s_old > s_run ? s_old : s_run;
    if (s > s_old) {
      for (int t = 0; t < off0; ++t) {
        uint8_t* row = row_ptr(c, blk, h, kv, t);
        for (int ch = 0; ch < c->D; ++ch) {
          float old_val = (float)mf_decode(f, row[ch]) * s_old;
          row[ch] = (uint8_t)mf_encode(f, old_val / s);
        }
      }
    }
  }
  *sp = s;
  for (int j = 0; j < n; ++j) {
    uint8_t* row = row_ptr(c, blk, h, kv, off0 + j);
    for (int ch = 0; ch < c->D; ++ch) {
      float v = in_value(x, in_dt, (size_t)(t0 + j) * tok_stride + (size_t)h * c->D + ch);
      row[ch] = (s > 0.0f) ? (uint8_t)mf_encode(f, v / s) : 0;
    }
  }
}

/* FP4 + outlier write of one run ([P1] steps 1-3).
 * Step 1, "per-channel magnitude norms", read as the L-infinity norm of each
 * channel over the tokens of the block's first write. Step 2, "dynamic variance
 * threshold (>= 3.2 sigma)", read as n_c >= mu + 3.2 sigma with mu, sigma the
 * mean and population standard deviation of the D channel norms, summed in fp64
 * in channel order; at most 4 outliers kept (largest norm first, ties to the
 * lower channel), stored ascending; their values go to the FP16 buffer. Step 3,
 * "normalized and quantized to FP4", read as one E4M3 scale per 16 channels of
 * a token (absmax / 6 over non-outlier channels) and E2M1 codes. */
static void write_fp4_run(const cache_t* c, const uint16_t* x, int in_dt, int t0, int n,
                          int blk, int off0, int h, int kv) {
  const int D = c->D;
  const size_t tok_stride = (size_t)c->H * D;
  uint8_t* idx = fp4_idx_ptr(c, blk, h, kv);
  if (off0 == 0) {
    float norm[128];
    for (int ch = 0; ch < D; ++ch) {
      float m = 0.0f;
      for (int j = 0; j < n; ++j) {
        float v = fabsf(in_value(x, in_dt, (size_t)(t0 + j) * tok_stride + (size_t)h * D + ch));
        if (v > m) m = v;
      }
      norm[ch] = m;
    }
    double s1 = 0.0, s2 = 0.0;
    for (int ch = 0; ch < D; ++ch) {
      double v = (double)norm[ch];
      s1 = s1 + v;
      s2 = s2 + v * v;
    }
    double mu = s1 / (double)D;
    double var = s2 / (double)D - mu * mu;
    if (var < 0.0) var = 0.0;
    double thr = mu + 3.2 * sqrt(var);
    int taken[128] = {0};
    int chosen[R_OUT];
    int nchosen = 0;
    for (int r = 0; r < R_OUT; ++r) {
      int best = -1;
      for (int ch = 0; ch < D; ++ch) {
        if (taken[ch] || !((double)norm[ch] >= thr)) continue;
        if (best < 0 || norm[ch] > norm[best]) best = ch;
      }
      if (best < 0) break;
      taken[best] = 1;
      chosen[nchosen++] = best;
    }
    /* ascending order */
    for (int i = 1; i < nchosen; ++i)
      for (int j = i; j > 0 && chosen[j - 1] > chosen[j]; --j) {
        int tmp = chosen[j];
        chosen[j] = chosen[j - 1];
        chosen[j - 1] = tmp;
      }
    for (int r = 0; r < IDX_STRIDE; ++r) idx[r] = (r < nchosen) ? (uint8_t)chosen[r] : 0xFF;
  }
  int is_out[128] = {0};
  int slot_ch[R_OUT];
  for (int r = 0; r < R_OUT; ++r) {
    slot_ch[r] = (idx[r] < D) ? idx[r] : -1;
    if (slot_ch[r] >= 0) is_out[slot_ch[r]] = 1;
  }
  for (int j = 0; j < n; ++j) {
    const int t = off0 + j;
    const size_t base = (size_t)(t0 + j) * tok_stride + (size_t)h * D;
    uint16_t* vals = fp4_val_ptr(c, blk, h, kv, t);
    for (int r = 0; r < R_OUT; ++r)
      vals[r] = (slot_ch[r] >= 0) ? (uint16_t)mf_encode(&F_FP16, in_value(x, in_dt, base + slot_ch[r])) : 0;
    uint8_t* sc = fp4_scale_ptr(c, blk, h, kv, t);
    for (int g = 0; g < D / GROUP; ++g) {
      float a = 0.0f;
      for (int ch = g * GROUP; ch < (g + 1) * GROUP; ++ch) {
        if (is_out[ch]) continue;
        float v = fabsf(in_value(x, in_dt, base + ch));
        if (v > a) a = v;
      }
      uint32_t scode = mf_encode(&F_E4M3, a / 6.0f);
      sc[g] = (uint8_t)scode;
      float sd = (float)mf_decode(&F_E4M3, scode);
      for (int ch = g * GROUP; ch < (g + 1) * GROUP; ++ch) {
        int code = 0;
        if (!is_out[ch] && sd != 0.0f) code = (int)mf_encode(&F_E2M1, in_value(x, in_dt, base + ch) / sd);
        fp4_set_code(c, blk, h, kv, t, ch, code);
      }
    }
  }
}

/* Cache write. Slot s -> block s/16, offset s%16 ([P3] PagedAttention). Runs:
 * token i continues token i-1 when both are valid, slot[i] == slot[i-1] + 1 and
 * slot[i] is not the first slot of a block. Runs are applied in token order. */
int oracle_kv_cache_write(const uint16_t* k, const uint16_t* v, int in_dt, int T,
                          const int32_t* slots, uint8_t* cache, uint8_t* scales,
                          uint8_t* oidx, uint8_t* oval, int kv_dt, int nb, int H, int D,
                          int32_t* err) {
  cache_t c = {kv_dt, nb, H, D, cache, scales, oidx, oval};
  const size_t tok_stride = (size_t)H * D;
  if (kv_dt == DT_FP16 || kv_dt == DT_BF16) {
    if (in_dt != kv_dt) return 1;
    for (int i = 0; i < T; ++i) {
      int s = slots[i];
      if (s < 0) continue;
      if ((int64_t)s >= (int64_t)nb * BS) {
        *err |= ERR_SLOT;
        continue;
      }
      for (int h = 0; h < H; ++h)
        for (int kv = 0; kv < 2; ++kv)
          memcpy(row_ptr(&c, s / BS, h, kv, s % BS), (kv ? v : k) + (size_t)i * tok_stride + (size_t)h * D,
                 (size_t)D * 2);
    }
    return 0;
  }
  int i = 0;
  while (i < T) {
    int s = slots[i];
    if (s < 0) {
      ++i;
      continue;
    }
    if ((int64_t)s >= (int64_t)nb * BS) {
      *err |= ERR_SLOT;
      ++i;
      continue;
    }
    if (i > 0) {
      int p = slots[i - 1];
      if (p >= 0 && (int64_t)p < (int64_t)nb * BS && p / BS == s / BS) *err |= ERR_RUN;
    }
    int n = 1;
    while (i + n < T) {
      int s2 = slots[i + n];
      if (s2 != s + n || s2 % BS == 0) break;
      ++n;
    }
    for (int h = 0; h < H; ++h)
      for (int kv = 0; kv < 2; ++kv) {
        const uint16_t* x = kv ? v : k;
        if (kv_dt == DT_E2M1)
          write_fp4_run(&c, x, in_dt, i, n, s / BS, s % BS, h, kv);
        else
          write_fp8_run(&c, x, in_dt, i, n, s / BS, s % BS, h, kv);
      }
    i += n;
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode attention                                                           */
/* ------------------------------------------------------------------------ */

/* Gather sequence b's tokens of KV head h through its block table and
 * dequantize them into contiguous fp64 arrays kd, vd [L][D] ([P3]
 * PagedAttention: logical block t/16 -> physical block table[t/16]). Tokens
 * of a block id outside [0, nb) are marked invalid (valid[t] = 0). */
void oracle_gather(const uint8_t* cache, const uint8_t* scales, const uint8_t* oidx,
                   const uint8_t* oval, int kv_dt, int nb, int H, int D,
                   const int32_t* table, int L, int h, double* kd, double* vd,
                   uint8_t* valid) {
  cache_t c = {kv_dt, nb, H, D, (uint8_t*)cache, (uint8_t*)scales, (uint8_t*)oidx, (uint8_t*)oval};
  for (int t = 0; t < L; ++t) {
    int blk = table[t / BS];
    valid[t] = (blk >= 0 && blk < nb);
    for (int ch = 0; ch < D; ++ch) {
      kd[(size_t)t * D + ch] = valid[t] ? dequant(&c, blk, h, 0, t % BS, ch) : 0.0;
      vd[(size_t)t * D + ch] = valid[t] ? dequant(&c, blk, h, 1, t % BS, ch) : 0.0;
    }
  }
}

/* softmax(scale * q K^T) V in fp64 over the valid tokens. out[D]. */
static void attend(const double* q, const double* kd, const double* vd, const uint8_t* valid,
                   int L, int D, double scale, double* out, double* sbuf) {
  double m = -INFINITY;
  for (int t = 0; t < L; ++t) {
    if (!valid[t]) continue;
    double dot = 0.0;
    for (int ch = 0; ch < D; ++ch) dot += q[ch] * kd[(size_t)t * D + ch];
    sbuf[t] = scale * dot;
    if (sbuf[t] > m) m = sbuf[t];
  }
  for (int ch = 0; ch < D; ++ch) out[ch] = 0.0;
  if (m == -INFINITY) return;
  double denom = 0.0;
  for (int t = 0; t < L; ++t) {
    if (!valid[t]) continue;
    double w = exp(sbuf[t] - m);
    denom += w;
    for (int ch = 0; ch < D; ++ch) out[ch] += w * vd[(size_t)t * D + ch];
  }
  for (int ch = 0; ch < D; ++ch) out[ch] /= denom;
}

/* Paged decode attention, fp64 output out[B][Hq][D]. Query head hq reads KV
 * head hq / (Hq / H). */
int oracle_paged_decode(const uint16_t* q, int q_dt, int B, int Hq, const uint8_t* cache,
                        const uint8_t* scales, const uint8_t* oidx, const uint8_t* oval,
                        int kv_dt, int nb, int H, int D, const int32_t* tables, int maxblk,
                        const int32_t* seq_lens, float scale, double* out, int32_t* err) {
  if (Hq % H != 0) return 1;
  const int G = Hq / H;
  int32_t flags = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : flags)
  for (int bh = 0; bh < B * H; ++bh) {
    const int b = bh / H, h = bh % H;
    const int L = seq_lens[b];
    double* ob = out + ((size_t)b * Hq + (size_t)h * G) * D;
    if (L < 0 || (int64_t)L > (int64_t)BS * maxblk || L == 0) {
      if (L != 0) flags |= ERR_SEQ_LEN;
      for (size_t i = 0; i < (size_t)G * D; ++i) ob[i] = 0.0;
      continue;
    }
    double* kd = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* vd = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* sb = (double*)malloc(sizeof(double) * (size_t)L);
    uint8_t* valid = (uint8_t*)malloc((size_t)L);
    double qd[128];
    oracle_gather(cache, scales, oidx, oval, kv_dt, nb, H, D, tables + (size_t)b * maxblk, L, h, kd, vd,
                  valid);
    for (int t = 0; t < L; ++t)
      if (!valid[t]) flags |= ERR_BLOCK_ID;
    for (int g = 0; g < G; ++g) {
      const size_t qoff = ((size_t)b * Hq + (size_t)h * G + g) * D;
      for (int ch = 0; ch < D; ++ch) qd[ch] = (double)in_value(q, q_dt, qoff + ch);
      attend(qd, kd, vd, valid, L, D, (double)scale, ob + (size_t)g * D, sb);
    }
    free(kd);
    free(vd);
    free(sb);
    free(valid);
  }
  *err |= flags;
  return 0;
}

/* Chunked-prefill attention ([P1] architecture diagram: prompts processed in
 * 512-token chunks; [P3] "Chunked prefill"). The qn = cu_q[b+1] - cu_q[b] query
 * tokens of sequence b are its last qn positions: query token i sits at
 * position p = seq_lens[b] - qn + i and attends to positions 0..p (causal), read
 * through the block table like decode. q and out: [cu_q[B]][Hq][D]. A sequence
 * with qn > seq_lens[b] or seq_lens[b] beyond its table is skipped (SEQ_LEN,
 * zero output rows). */
int oracle_paged_prefill(const uint16_t* q, int q_dt, const int32_t* cu_q, int B, int Hq,
                         const uint8_t* cache, const uint8_t* scales, const uint8_t* oidx,
                         const uint8_t* oval, int kv_dt, int nb, int H, int D, const int32_t* tables,
                         int maxblk, const int32_t* seq_lens, float scale, double* out, int32_t* err) {
  if (Hq % H != 0) return 1;
  const int G = Hq / H;
  int32_t flags = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : flags)
  for (int bh = 0; bh < B * H; ++bh) {
    const int b = bh / H, h = bh % H;
    const int L = seq_lens[b];
    const int qn = cu_q[b + 1] - cu_q[b];
    if (qn <= 0) continue;
    if (L < 0 || (int64_t)L > (int64_t)BS * maxblk || qn > L) {
      flags |= ERR_SEQ_LEN;
      for (int i = 0; i < qn; ++i)
        for (size_t e = 0; e < (size_t)G * D; ++e)
          out[((size_t)(cu_q[b] + i) * Hq + (size_t)h * G) * D + e] = 0.0;
      continue;
    }
    double* kd = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* vd = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* sb = (double*)malloc(sizeof(double) * (size_t)L);
    uint8_t* valid = (uint8_t*)malloc((size_t)L);
    double qd[128];
    oracle_gather(cache, scales, oidx, oval, kv_dt, nb, H, D, tables + (size_t)b * maxblk, L, h, kd, vd,
                  valid);
    for (int t = 0; t < L; ++t)
      if (!valid[t]) flags |= ERR_BLOCK_ID;
    for (int i = 0; i < qn; ++i) {
      const int pos = L - qn + i;
      for (int g = 0; g < G; ++g) {
        const size_t row = ((size_t)(cu_q[b] + i) * Hq + (size_t)h * G + g) * D;
        for (int ch = 0; ch < D; ++ch) qd[ch] = (double)in_value(q, q_dt, row + ch);
        attend(qd, kd, vd, valid, pos + 1, D, (double)scale, out + row, sb);
      }
    }
    free(kd);
    free(vd);
    free(sb);
    free(valid);
  }
  *err |= flags;
  return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
