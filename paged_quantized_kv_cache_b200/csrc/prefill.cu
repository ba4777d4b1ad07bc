// prefill.cu -- chunked-prefill attention over the paged, quantized KV cache,
// on the sm_100a tensor cores (tcgen05, accumulators in tensor memory).
//
// Method: "vLLM" glossary, "Chunked prefill" (a long prompt is processed in
// chunks) and "PagedAttention" (K/V read through the block table); "vLLM 0.7
// Ships Unified KV Cache Compression", architecture diagram (512-token chunks)
// and step 4 (the attention kernel reads the compressed codes and the fp16
// outlier channels together). The q_len query tokens of a sequence are its last
// q_len cached positions (the chunk is written to the cache first); query token
// i at position p attends to positions 0..p.
//
// Work decomposition. One CTA per (sequence, KV head, pair of 128-row tiles); a
// row is (query token, query head of the GQA group), so a tile holds 128 / G
// query tokens. Warps have one role each:
//   two compute warpgroups, one row per thread (its S, P and O rows live in
//     tensor-memory lane r of the warpgroup's 256 columns): online softmax;
//   a producer warp: refills each stage of a 4-deep ring as soon as it is
//     released (by the MMA warps' commits after the last products reading it, or
//     once its raw codes are dequantized);
//   for quantized caches, a dequantization warpgroup: turns each tile's raw
//     codes into f16 operands as soon as the products that read the previous
//     contents of its operand buffers are done;
//   an MMA warp per warpgroup: issues its tensor-core products and commits
//     each to an mbarrier, so no compute warp waits on a barrier with the
//     others, and neither warpgroup's products wait for the other's P.
// Per KV tile t of 64 tokens (4 cache blocks) and warpgroup:
//   S(t) = Q K(t)^T        tcgen05.mma M=128 N=64 (A, B in shared memory),
//                          into one of two S buffers in tensor memory
//   softmax of S(t)        one row per thread, no shuffles, lazy rescale of O
//   P(t) -> tensor memory  over the S(t) columns (16-bit, two per column;
//                          P = P_hi + P_lo for bf16), then one arrival per warp
//   O += P(t) V(t)         tcgen05.mma M=128 N=D, A = P from tensor memory
// The MMA warp issues S(t + 2) into a buffer as soon as PV(t) has read the P
// it held, so the scores of a warpgroup's next tile are always computed while
// it exponentiates the current one. Operands in shared memory are
// 128-byte-swizzled tiles: 16-bit K/V land there directly by TMA; FP8 / FP4
// tiles are fetched raw (one bulk copy per block plus its scales and outlier
// buffers) and dequantized into f16 operands. FP8 scales stay out of the
// operands: the K scale multiplies S, the V scale multiplies P relative to
// the largest V scale seen so far (O is kept in units of it). FP4 operands are
// exact in f16 (E2M1 x E4M3 and the fp16 outlier values).
#include <atomic>
#include <cfloat>

#include "prefill.cuh"
#include "tcgen05.cuh"

namespace pqkv {

namespace {

constexpr int kM = 128;        // rows (query token, head) per warpgroup tile
constexpr int kN = 64;         // KV tokens per tile (4 blocks)
constexpr int kWG = 128;       // threads of a compute warpgroup: one row (TMEM lane) per thread
constexpr float kLazy = 8.f;   // O is rescaled only when a row max grows by more (log2 units)
constexpr unsigned kFull = 0xFFFFFFFFu;

template <int KVF, int D>
struct PrefillGeom {
  static constexpr bool k16 = (KVF == PQKV_DTYPE_FP16 || KVF == PQKV_DTYPE_BF16);
  static constexpr bool kFp8 = (KVF == PQKV_DTYPE_FP8_E4M3 || KVF == PQKV_DTYPE_FP8_E5M2);
  static constexpr bool kFp4 = (KVF == PQKV_DTYPE_FP4_E2M1);
  // Two compute warpgroups per CTA, each on its own 128-row query tile, sharing
  // the K/V stages (one issues while the other stalls; a K/V tile serves 256
  // rows). Quantized tiles are dequantized by both together.
  static constexpr int NWG = 2;
  static constexpr int kStages = 4;                // KV tiles in flight (shared memory)
  // quantized caches: a dequantization warpgroup; 128 threads take the 64 x D/8
  // operand chunks of a tile in a fixed number of rounds, unrolled so that the
  // chains of several chunks overlap (16 warps in all: at most 4 per scheduler,
  // so 128 registers a thread fit)
  static constexpr int kDeqWarps = k16 ? 0 : 4;
  static constexpr int kDeqThreads = 32 * kDeqWarps;
  // compute warpgroups + a producer warp + an MMA warp per warpgroup (+ dequantization)
  static constexpr int kThreads = NWG * kWG + 32 + 32 * NWG + kDeqThreads;
  static constexpr int NB = D / 64;                // 128-byte boxes per operand row
  static constexpr int kQBytes = NB * kM * 128;    // Q operand of one warpgroup [box][128 rows][128 B]
  static constexpr int kOpBytes = NB * kN * 128;   // one K or V operand tile [box][64 rows][128 B]
  // bf16 operands: P = P_hi + P_lo, both rounded to bf16, keeps ~16 significant
  // bits of the probabilities (a bf16 P alone errs by up to |v| 2^-9, too much
  // for the 2e-3 tolerance); f16 operands (fp16, FP8, FP4 caches) take a single
  // f16 P (|v| 2^-11 at most). P lives in tensor memory, over the columns of
  // the S tile it came from (32 columns per part).
  static constexpr bool kSplitP = (KVF == PQKV_DTYPE_BF16);
  static constexpr int kRawTile = 32 * row_bytes(KVF, D);  // one block's K|V codes
  static constexpr int kScaleBytes = kFp8 ? 16 : (kFp4 ? 2 * 16 * (D / 16) : 0);
  static constexpr int kValBytes = kFp4 ? 2 * 16 * 4 * 2 : 0;
  static constexpr int kIdxBytes = kFp4 ? 16 : 0;
  static constexpr int kSide = kScaleBytes + kValBytes + kIdxBytes;
  static constexpr int kRawStage = k16 ? 2 * kOpBytes : 4 * (kRawTile + kSide);
  static constexpr int kStageBytes = (kRawStage + 1023) / 1024 * 1024;
  static constexpr int kKops = k16 ? 0 : 2;        // dequantized K tiles (S of tile t-1 may still read one)
  static constexpr int kVops = k16 ? 0 : 3;        // dequantized V tiles (PV of tile t-2 may still read one)
  static constexpr int oQ = 0;
  static constexpr int oStage = oQ + NWG * kQBytes;
  static constexpr int oKop = oStage + kStages * kStageBytes;
  static constexpr int oVop = oKop + kKops * kOpBytes;
  static constexpr int oMisc = oVop + kVops * kOpBytes;
  static constexpr int kMiscBytes = 512;
  static constexpr int kSmem = oMisc + kMiscBytes + 1024;  // + alignment slack
  static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
  // per warpgroup 256 columns: O at [0, D), S buffers at D and D + 64
  static constexpr uint32_t kTmemCols = 256 * NWG;
};

__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint32_t to_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Barrier of the N dequantization threads (named barrier 1), and its and-reduction.
template <int N>
__device__ __forceinline__ void deq_sync() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }
template <int N>
__device__ __forceinline__ bool deq_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(N)
      : "memory");
  return r != 0;
}

// Packed pairs of fp32 operations (two lanes of IEEE fp32 arithmetic, rounded to
// nearest, in one instruction): (d0, d1) = (a0, a1) op (b0, b1) [+ (c0, c1)].
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void sub2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// E4M3 scale byte -> f16x2 (s, s).
__device__ __forceinline__ __half2 scale2(uint32_t byte) {
  const uint32_t r = dec_fp8x2<PQKV_DTYPE_FP8_E4M3>(byte | (byte << 8));
  return *reinterpret_cast<const __half2*>(&r);
}

__device__ __forceinline__ uint32_t hmul2u(uint32_t a, __half2 s) {
  __half2 x = __hmul2(*reinterpret_cast<const __half2*>(&a), s);
  return *reinterpret_cast<uint32_t*>(&x);
}

}  // namespace

template <int KVF, int D, bool QBF16>
__global__ void __launch_bounds__(PrefillGeom<KVF, D>::kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap, const PrefillParams p) {
  using Gm = PrefillGeom<KVF, D>;
  constexpr int NWG = Gm::NWG, kStages = Gm::kStages;
  constexpr bool kBfMma = (KVF == PQKV_DTYPE_BF16);  // operand type: bf16 for a bf16 cache, else f16
  constexpr uint32_t kIdescS = tc::f16_idesc(kBfMma, kM, kN, false);
  constexpr uint32_t kIdescPV = tc::f16_idesc(kBfMma, kM, D, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sStage = smem + Gm::oStage;
  uint8_t* sKop = smem + Gm::oKop;
  uint8_t* sVop = smem + Gm::oVop;
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + Gm::oMisc);  // [kStages] tile landed
  uint64_t* bar_empty = bar_full + kStages;                             // [kStages] stage free again
  uint64_t* bar_s = bar_empty + kStages;     // [NWG][2] S(t) computed (buffer t % 2)
  uint64_t* bar_p = bar_s + 2 * NWG;         // [NWG][2] P(t) in tensor memory (one arrival per warp)
  uint64_t* bar_pv = bar_p + 2 * NWG;        // [NWG][2] PV(t) computed
  uint64_t* bar_op = bar_pv + 2 * NWG;       // [4] quantized: operands, mask and scales of tile t ready
  uint64_t* bar_kfree = bar_op + 4;          // [2] quantized: S(t) of every warpgroup done (kop[t % 2])
  uint64_t* bar_vfree = bar_kfree + 2;       // [3] quantized: PV(t) of every warpgroup done (vop[t % 3])
  uint64_t* bar_drain = bar_vfree + 3;       // [NWG] every product an MMA warp issued has completed
  float* tile_sk = reinterpret_cast<float*>(bar_drain + NWG);  // [4][4] FP8 K scales of tile t % 4
  float* tile_sv = tile_sk + 16;                               // [4][4] FP8 V scales
  volatile int* op_mask = reinterpret_cast<volatile int*>(tile_sv + 16);  // [4] quantized: blocks of tile t % 4
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(op_mask) + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* n_issued_slot = reinterpret_cast<int*>(tmem_slot + 2);
  volatile int* stage_mask = reinterpret_cast<volatile int*>(tmem_slot + 4);  // [kStages] blocks fetched

  asm volatile("griddepcontrol.wait;" ::: "memory");  // the chunk's K/V may come from the previous kernel
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int G = p.G, TOK = kM / G;
  const int ctas = (p.tiles_per_seq + NWG - 1) / NWG;  // CTAs per sequence
  const int b = blockIdx.x / ctas;
  const int mt0 = NWG * (ctas - 1 - (int)(blockIdx.x % ctas));  // first query tile; long ones first
  const int q0 = p.cu_q[b], qn = p.cu_q[b + 1] - q0;
  const int L = p.seq_lens[b];
  if (mt0 == 0 && h == 0 && tid == 0 && qn > p.tiles_per_seq * TOK)
    raise_flag(p.err, PQKV_DEVERR_SEQ_LEN);  // rows past max_q_len are not computed
  if (qn <= 0 || mt0 * TOK >= qn) return;
  const bool is_compute = tid < NWG * kWG;
  const bool is_producer = warp == NWG * 4;
  const bool is_mma = warp > NWG * 4 && warp <= NWG * 4 + NWG, is_deq = warp > NWG * 4 + NWG;
  const int wg = is_compute ? tid / kWG : 0;
  const int r = tid % kWG;                           // row of this thread in its warpgroup's tile
  const int i0 = (mt0 + wg) * TOK;                   // first query token of the warpgroup's tile
  const int my_i = i0 + r / G, my_n = r % G;
  const bool row_ok = is_compute && my_i < qn && i0 < p.tiles_per_seq * TOK;
  const size_t orow = ((size_t)(q0 + (row_ok ? my_i : 0)) * p.Hq + (size_t)h * G + my_n) * D;
  if (L < 0 || L > kBlock * p.maxblk || qn > L) {
    if (mt0 == 0 && h == 0 && tid == 0) raise_flag(p.err, PQKV_DEVERR_SEQ_LEN);
    if (row_ok) {
      uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.out) + orow * 2);
      for (int c = 0; c < D / 8; ++c) o[c] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const int pos0 = L - qn;                          // position of query token 0
  const int my_pos = pos0 + my_i;                   // this row attends to [0, my_pos]
  // the CTA reads positions up to its last row: every warpgroup walks all its tiles
  const int n_kv = pos0 + min(min(mt0 + NWG, p.tiles_per_seq) * TOK, qn);
  const int T = (n_kv + kN - 1) / kN;
  const int32_t* table = p.block_tables + (size_t)b * p.maxblk;

  // ---- setup: tensor memory, barriers, Q tiles ----
  if (warp == 0) tc::tmem_alloc(tmem_slot, Gm::kTmemCols);
  if (tid == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], Gm::k16 ? NWG : 1);  // 16-bit: each MMA warp's commit; else dequantized
    }
    for (int i = 0; i < 2 * NWG; ++i) {
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_p[i], 4);
      mbar_init(&bar_pv[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bar_op[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&bar_kfree[i], NWG);
    for (int i = 0; i < 3; ++i) mbar_init(&bar_vfree[i], NWG);
    for (int i = 0; i < NWG; ++i) mbar_init(&bar_drain[i], 1);
    *abort_flag = 0;
    *n_issued_slot = 0;
    fence_mbar_init();
  }
  if constexpr (Gm::k16)
    if (tid == NWG * kWG) prefetch_tensormap(&tmap);
  // softmax scale in log2 units of this thread's row, times 2^e when the row's
  // bf16 query was scaled by 2^-e before narrowing to f16 (quantized caches)
  float sl2 = p.scale_log2;
  if (is_compute) {
    // row r of the warpgroup's Q tile, converted to the operand type, 16-byte chunks swizzled
    uint8_t* sQ = smem + Gm::oQ + wg * Gm::kQBytes;
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.q) + orow * 2);
    float qmul = 1.f;
    if constexpr (!Gm::k16 && QBF16) {
      // the power of two 2^-e that brings the row's largest |q| into
      // [2^13, 2^14): exact, and far from both ends of the f16 range
      float mx = 0.f;
      if (row_ok) {
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = __ldg(src + c);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
        }
      }
      const int ex = (mx > 0.f && mx <= FLT_MAX) ? ilogbf(mx) - 13 : 0;
      qmul = ldexpf(1.f, -ex);
      sl2 = p.scale_log2 * ldexpf(1.f, ex);
    }
#pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row_ok) v = __ldg(src + c);
      if constexpr (!Gm::k16 && QBF16) {  // bf16 query -> f16 operand, scaled by 2^-e
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = to_f16x2(__uint_as_float(w[i] << 16) * qmul, __uint_as_float(w[i] & 0xFFFF0000u) * qmul);
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const int bx = c >> 3, ch = c & 7;
      *reinterpret_cast<uint4*>(sQ + bx * (kM * 128) + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
    }
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  int n_prepared = 0;  // KV tiles this thread waited for, while no wait had given up

  if (is_producer) {
    // ================= producer warp: KV tiles into the stage ring =================
    if (lane == 0) {
      int t = 0;
      for (; t < T; ++t) {
        const int s = t % kStages;
        if (t >= kStages &&
            !mbar_wait_bounded(&bar_empty[s], (uint32_t)((t / kStages) - 1) & 1u, p.timeout_ns))
          break;
        if (*abort_flag) break;
        uint8_t* st = sStage + s * Gm::kStageBytes;
        int ids[4];
        int mask = 0;
        uint32_t bytes = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ids[j] = -1;
          const int blk = 4 * t + j;
          if (blk * kBlock < n_kv) {
            const int id = __ldg(table + blk);
            if (id >= 0 && id < p.nb) {
              ids[j] = id;
              mask |= 1 << j;
              bytes += Gm::k16 ? 2u * Gm::NB * kBlock * 128u : (uint32_t)(Gm::kRawTile + Gm::kSide);
            } else {
              raise_flag(p.err, PQKV_DEVERR_BLOCK_ID);
            }
          }
        }
        stage_mask[s] = mask;  // published to the consumers by the stage's barrier
        mbar_arrive_expect_tx(&bar_full[s], bytes);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (ids[j] < 0) continue;
          const size_t pair = (size_t)ids[j] * p.Hkv + h;
          if constexpr (Gm::k16) {
            const int y = (int)pair * 32;
#pragma unroll
            for (int bx = 0; bx < Gm::NB; ++bx) {
              tma_load_2d(st + bx * kN * 128 + j * kBlock * 128, &tmap, bx * 64, y, &bar_full[s]);
              tma_load_2d(st + Gm::kOpBytes + bx * kN * 128 + j * kBlock * 128, &tmap, bx * 64, y + 16,
                          &bar_full[s]);
            }
          } else {
            bulk_load(st + j * Gm::kRawTile, p.cache + pair * Gm::kRawTile, Gm::kRawTile, &bar_full[s]);
            uint8_t* side = st + 4 * Gm::kRawTile + j * Gm::kSide;
            if constexpr (Gm::kFp8) {
              bulk_load(side, p.scales + pair * 16, 16, &bar_full[s]);
            } else {
              bulk_load(side, p.scales + pair * Gm::kScaleBytes, Gm::kScaleBytes, &bar_full[s]);
              bulk_load(side + Gm::kScaleBytes, p.oval + pair * Gm::kValBytes, Gm::kValBytes, &bar_full[s]);
              bulk_load(side + Gm::kScaleBytes + Gm::kValBytes, p.oidx + pair * 16, 16, &bar_full[s]);
            }
          }
        }
      }
      *n_issued_slot = t;
    }
  } else if (is_mma) {
    // ================= MMA warp w: every tensor-core product of warpgroup w =================
    // Order per KV tile t: PV(t) once the warpgroup's P(t) is in tensor memory,
    // then S(t + 2) into the buffer P(t) occupied, once PV(t) has read it.
    // S(0) and S(1) are issued up front, so the warpgroup finds the scores of
    // its next tile computed. One MMA warp per warpgroup keeps the two chains
    // independent: neither waits for the other's P (they share the tensor pipe).
    const int w = warp - (NWG * 4 + 1);
    if (lane == 0) {
      bool good = true;
      // operands of tile t ready: 16-bit K/V landed; quantized tiles dequantized
      auto ready = [&](int t) -> bool {
        if constexpr (Gm::k16)
          return mbar_wait_bounded(&bar_full[t % kStages], (uint32_t)(t / kStages) & 1u, p.timeout_ns);
        else
          return mbar_wait_bounded(&bar_op[t & 3], (uint32_t)(t >> 2) & 1u, p.timeout_ns);
      };
      auto issue_s = [&](int t) {
        tc::fence_after_sync();
        const uint32_t d = tmem + 256u * w + D + 64 * (t & 1);
        const uint8_t* kop = Gm::k16 ? sStage + (t % kStages) * Gm::kStageBytes : sKop + (t & 1) * Gm::kOpBytes;
        const uint32_t qa = smem_u32(smem + Gm::oQ + w * Gm::kQBytes), ka = smem_u32(kop);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = tc::sw128_desc(qa + (kk >> 2) * (kM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(ka + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_ss(d, a, bd, kIdescS, kk > 0);
        }
        tc::commit(&bar_s[2 * w + (t & 1)]);
        if constexpr (!Gm::k16) tc::commit(&bar_kfree[t & 1]);  // the K operand buffer may be refilled
      };
      auto issue_pv = [&](int t) {
        tc::fence_after_sync();
        const uint8_t* vop = Gm::k16 ? sStage + (t % kStages) * Gm::kStageBytes + Gm::kOpBytes
                                     : sVop + (t % 3) * Gm::kOpBytes;
        const uint32_t o = tmem + 256u * w, pa = o + D + 64 * (t & 1), va = smem_u32(vop);
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk) {
          const uint64_t bd = tc::sw128_desc(va + kk * 2048, kN * 128, 1024);
          tc::mma_ts(o, pa + kk * 8, bd, kIdescPV, !(t == 0 && kk == 0));
          if constexpr (Gm::kSplitP) tc::mma_ts(o, pa + 32 + kk * 8, bd, kIdescPV, true);
        }
        tc::commit(&bar_pv[2 * w + (t & 1)]);
        if constexpr (!Gm::k16) tc::commit(&bar_vfree[t % 3]);  // the V operand buffer may be refilled
      };
      for (int t = 0; t < min(2, T) && good; ++t) {
        good = ready(t);
        if (good) issue_s(t);
      }
      for (int t = 0; t < T && good; ++t) {
        good = mbar_wait_bounded(&bar_p[2 * w + (t & 1)], (uint32_t)(t >> 1) & 1u, p.timeout_ns);
        if (!good) break;
        issue_pv(t);
        // a 16-bit stage holds the operands themselves: free once S(t) and PV(t)
        // of every warpgroup are done (one commit per MMA warp)
        if constexpr (Gm::k16) tc::commit(&bar_empty[t % kStages]);
        if (t + 2 < T) {
          good = ready(t + 2) &&
                 mbar_wait_bounded(&bar_pv[2 * w + (t & 1)], (uint32_t)(t >> 1) & 1u, p.timeout_ns);
          if (good) issue_s(t + 2);
        }
      }
      if (!good) {
        *abort_flag = 1;
        raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
      }
      // every product issued completes before tensor memory is released
      tc::commit(&bar_drain[w]);
      if (!mbar_wait_bounded(&bar_drain[w], 0, p.drain_ns)) raise_flag(p.err, PQKV_DEVERR_DRAIN);
    }
  } else if (is_deq) {
    // ================= dequantization warps (quantized caches) =================
    // Tile t: raw codes landed, the operand buffers free again (S(t - 2) read
    // kop[t % 2], PV(t - 3) read vop[t % 3], for both warpgroups), then the
    // codes become f16 operands; bar_op[t % 4] hands them, the tile's block
    // mask and FP8 scales to the MMA and compute warps, and the raw stage goes
    // back to the producer. The dequantization warps leave together, at a consensus.
    if constexpr (!Gm::k16) {
      const int dq = tid - (NWG * 4 + 1 + NWG) * 32;  // 0 .. kDeqThreads - 1
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const int s = t % kStages;
        ok = mbar_wait_bounded(&bar_full[s], (uint32_t)(t / kStages) & 1u, p.timeout_ns) && ok;
        if (ok) ++n_prepared;  // counted up to the first wait that gave up: the drain covers the rest
        if (t >= 2) ok = mbar_wait_bounded(&bar_kfree[t & 1], (uint32_t)((t >> 1) - 1) & 1u, p.timeout_ns) && ok;
        if (t >= 3) ok = mbar_wait_bounded(&bar_vfree[t % 3], (uint32_t)((t / 3) - 1) & 1u, p.timeout_ns) && ok;
        ok = deq_all<Gm::kDeqThreads>(ok);
        if (!ok) break;
        // blocks of the tile that were fetched, as the producer left them beside the stage
        const int mask = stage_mask[s];
        const int base = t * kN;
        uint8_t* st = sStage + s * Gm::kStageBytes;
        uint8_t* kop = sKop + (t & 1) * Gm::kOpBytes;
        uint8_t* vop = sVop + (t % 3) * Gm::kOpBytes;
        constexpr int CPR = D / 8;  // 16-byte operand chunks per row
        static_assert(kN * CPR % Gm::kDeqThreads == 0, "whole rounds");
        constexpr int kRounds = kN * CPR / Gm::kDeqThreads;  // a compile-time count: fully unrolled
#pragma unroll
        for (int k = 0; k < kRounds; ++k) {
          const int u = dq + k * Gm::kDeqThreads;
          const int rr = u / CPR, c = u % CPR, j = rr >> 4, tr = rr & 15;
          const bool okr = ((mask >> j) & 1) && base + rr < L;
          uint32_t kf[4] = {0, 0, 0, 0}, vf[4] = {0, 0, 0, 0};
          if (okr) {
            const uint8_t* tile = st + j * Gm::kRawTile;
            if constexpr (Gm::kFp8) {
              const uint2 kc = *reinterpret_cast<const uint2*>(tile + tr * D + 8 * c);
              const uint2 vc = *reinterpret_cast<const uint2*>(tile + (16 + tr) * D + 8 * c);
              kf[0] = dec_fp8x2<KVF>(kc.x);
              kf[1] = dec_fp8x2<KVF>(kc.x >> 16);
              kf[2] = dec_fp8x2<KVF>(kc.y);
              kf[3] = dec_fp8x2<KVF>(kc.y >> 16);
              vf[0] = dec_fp8x2<KVF>(vc.x);
              vf[1] = dec_fp8x2<KVF>(vc.x >> 16);
              vf[2] = dec_fp8x2<KVF>(vc.y);
              vf[3] = dec_fp8x2<KVF>(vc.y >> 16);
            } else {
              const uint8_t* side = st + 4 * Gm::kRawTile + j * Gm::kSide;
              constexpr int SPR = D / 16;  // scale bytes per token row
              // K: row tr, channels 8c..8c+7 = 4 bytes, channel 2i in the low nibble
              dec_e2m1x8(*reinterpret_cast<const uint32_t*>(tile + tr * (D / 2) + 4 * c), kf);
              // V: token-pair rows; this token's nibble of channels 8c..8c+7
              const int hh = (8 * c) / (D / 2);
              const int pr = tr < 8 ? (tr & ~1) : (((tr - 8) & ~1) + 1);
              const uint2 wv =
                  *reinterpret_cast<const uint2*>(tile + (16 + 8 * hh + pr) * (D / 2) + (8 * c) % (D / 2));
              const uint32_t x0 = ((tr & 1) ? (wv.x >> 4) : wv.x) & 0x0F0F0F0Fu;
              const uint32_t x1 = ((tr & 1) ? (wv.y >> 4) : wv.y) & 0x0F0F0F0Fu;
              dec_e2m1x8(prmt(x0 | (x0 >> 4), x1 | (x1 >> 4), 0x6420u), vf);
              const __half2 sk = scale2(side[tr * SPR + (c >> 1)]);
              const __half2 sv = scale2(side[16 * SPR + tr * SPR + (c >> 1)]);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                kf[i] = hmul2u(kf[i], sk);
                vf[i] = hmul2u(vf[i], sv);
              }
            }
          }
          const uint32_t off = (c >> 3) * (kN * 128) + rr * 128 + (((c & 7) ^ (rr & 7)) << 4);
          *reinterpret_cast<uint4*>(kop + off) = make_uint4(kf[0], kf[1], kf[2], kf[3]);
          *reinterpret_cast<uint4*>(vop + off) = make_uint4(vf[0], vf[1], vf[2], vf[3]);
        }
        if constexpr (Gm::kFp4) {
          // outlier channels (their codes are 0): write the fp16 values over them;
          // item = (block j, K|V, slot, eighth of the tokens)
          deq_sync<Gm::kDeqThreads>();
#pragma unroll
          for (int k = 0; k < 256 / Gm::kDeqThreads; ++k) {
            const int gt = dq + k * Gm::kDeqThreads;
            const int j = gt >> 6, kv = (gt >> 5) & 1, slot = (gt >> 3) & 3, part = gt & 7;
            if ((mask >> j) & 1) {
              const uint8_t* side = st + 4 * Gm::kRawTile + j * Gm::kSide;
              const int ch = side[Gm::kScaleBytes + Gm::kValBytes + 8 * kv + slot];
              if (ch < D) {
                const uint16_t* val = reinterpret_cast<const uint16_t*>(side + Gm::kScaleBytes) + kv * 64;
                uint8_t* op = kv ? vop : kop;
                const int c = ch >> 3;
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4) {
                  const int tr = 2 * part + q4, rr = 16 * j + tr;
                  if (base + rr < L)
                    *reinterpret_cast<uint16_t*>(op + (c >> 3) * (kN * 128) + rr * 128 + (((c & 7) ^ (rr & 7)) << 4) +
                                                 (ch & 7) * 2) = val[tr * 4 + slot];
                }
              }
            }
          }
        }
        if constexpr (Gm::kFp8) {
          if (dq < 4) {
            const bool okb = (mask >> dq) & 1;
            const float* sc = reinterpret_cast<const float*>(st + 4 * Gm::kRawTile + dq * Gm::kSide);
            tile_sk[(t & 3) * 4 + dq] = okb ? sc[0] : 0.f;
            tile_sv[(t & 3) * 4 + dq] = okb ? sc[1] : 0.f;
          }
        }
        if (dq == 0) op_mask[t & 3] = mask;
        tc::fence_smem_to_async();
        deq_sync<Gm::kDeqThreads>();  // every thread's part is written
        if (dq == 0) {
          mbar_arrive(&bar_empty[s]);  // a raw stage is free as soon as it is dequantized
          mbar_arrive(&bar_op[t & 3]);
        }
      }
      if (!ok && dq == 0) {
        *abort_flag = 1;
        raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
      }
    }
  } else if (is_compute) {
    // ================= compute warpgroup wg: one row per thread =================
    const uint32_t t_row = tmem + 256u * wg + ((uint32_t)(32 * (warp & 3)) << 16);
    uint64_t* my_s = bar_s + 2 * wg;
    uint64_t* my_p = bar_p + 2 * wg;
    uint64_t* my_pv = bar_pv + 2 * wg;
    bool ok = true;  // no wait of this thread has timed out
    bool aborted = false;
    int mask_cur = 0, mask_next = 0;  // blocks of tile t / t + 1 holding data

    // ---- 16-bit caches: KV tile t landed, V rows without data zeroed; returns its block mask ----
    auto prepare = [&](int t) -> int {
      const int s = t % kStages;
      ok = mbar_wait_bounded(&bar_full[s], (uint32_t)(t / kStages) & 1u, p.timeout_ns) && ok;
      if (ok) ++n_prepared;  // counted up to the first wait that gave up: the drain covers the rest
      // blocks of the tile that were fetched, as the producer left them beside
      // the stage (after a timeout the value may be stale: it is the same for
      // every thread, and the results are not used then)
      const int mask = stage_mask[s];
      const int base = t * kN;
      uint8_t* st = sStage + s * Gm::kStageBytes;
      if constexpr (Gm::k16) {
        // V rows without valid data (past the sequence, or a block not loaded)
        // are zeroed: P is 0 there, and 0 x NaN would poison O. Each warpgroup
        // zeroes before its own P(t) is handed over (the same zeros), so the
        // product PV(t) of each warpgroup follows its own zeroing.
        if (mask != 0xF || base + kN > L) {
          for (int u = r; u < kN * Gm::NB * 8; u += kWG) {
            const int rr = u / (Gm::NB * 8), k = u % (Gm::NB * 8);
            if (((mask >> (rr >> 4)) & 1) && base + rr < L) continue;
            *reinterpret_cast<uint4*>(st + Gm::kOpBytes + (k >> 3) * kN * 128 + rr * 128 + ((k & 7) << 4)) =
                make_uint4(0, 0, 0, 0);
          }
          tc::fence_smem_to_async();
        }
      }
      return mask;
    };

    // ---- main loop ----
    // A warp leaves when one of its threads' waits gave up (tensor-memory loads
    // and stores are collective over the warp, so the decision is too); no
    // barrier spans warps inside the loop. S(t) done implies PV(t - 2) done
    // (its MMA warp issues S(t) into the buffer P(t - 2) occupied only then).
    auto leave = [&]() -> bool { return !__all_sync(kFull, ok); };
    float m = -INFINITY, l = 0.f, vref = 0.f;
    float rvref = 0.f;  // FP8: 1 / vref (0 while vref is 0), recomputed only when vref grows
    if constexpr (Gm::k16) {
      mask_next = prepare(0);
      if (leave()) aborted = true;
    }

    for (int t = 0; t < T && !aborted; ++t) {
      if constexpr (Gm::k16) {
        mask_cur = mask_next;
        if (t + 1 < T) mask_next = prepare(t + 1);
      }
      ok = mbar_wait_bounded(&my_s[t & 1], (uint32_t)(t >> 1) & 1u, p.timeout_ns) && ok;
      // quantized: the tile's block mask and FP8 scales, left by the dequantization
      if constexpr (!Gm::k16) ok = mbar_wait_bounded(&bar_op[t & 3], (uint32_t)(t >> 2) & 1u, p.timeout_ns) && ok;
      if (leave()) {
        aborted = true;
        break;
      }
      if constexpr (!Gm::k16) mask_cur = op_mask[t & 3];
      tc::fence_after_sync();

      // scores of this row
      const uint32_t t_s = t_row + D + 64 * (t & 1);
      uint32_t sv[64];
      tc::tmem_ld64(t_s, sv);
      const int mask = mask_cur;
      // no column of this tile is masked for any row of the warpgroup: all 4
      // blocks valid and the tile ends at or before the first row's position
      // (rows past the chunk keep a zero query and are never stored)
      const bool full = mask == 0xF && t * kN + kN - 1 <= pos0 + i0;
      // raw scores; the log2-domain scale of block j (softmax scale, times the
      // FP8 K scale of the block) is applied in the exponent's FMA. A block
      // with no data has K scale 0 and all its scores masked (-inf): it takes
      // scale 1 so that no 0 x inf arises; an all-zero K block has scores of
      // exactly 0, whose logit is 0 with any scale.
      float vs[4] = {1.f, 1.f, 1.f, 1.f};
      float cj[4] = {sl2, sl2, sl2, sl2};
      if constexpr (Gm::kFp8) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float k = tile_sk[(t & 3) * 4 + j];
          cj[j] = sl2 * (k > 0.f ? k : 1.f);
          vs[j] = tile_sv[(t & 3) * 4 + j];
        }
      }
      float xs[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) xs[c] = __uint_as_float(sv[c]);
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (t * kN + c > my_pos || !((mask >> (c >> 4)) & 1) || !row_ok) xs[c] = -INFINITY;
      }
      float mx;
      {
        // max of each half-block in 8 chains, then of each block times its scale
        // (positive: the max commutes with it; -inf stays -inf)
        float mp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mp[i] = xs[8 * i];
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c & 7) mp[c >> 3] = fmaxf(mp[c >> 3], xs[c]);
        mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float mb = fmaxf(mp[2 * j], mp[2 * j + 1]);
          if (mb != -INFINITY) mx = fmaxf(mx, mb * cj[j]);
        }
      }
      float fm = 1.f;  // rescale of l and O for a larger row max
      if (mx > m + kLazy) {
        fm = ex2(m - mx);  // 0 when m was -inf
        m = mx;
      }
      float fv = 1.f;  // FP8: O moves to units of a larger V scale (same on every thread)
      if constexpr (Gm::kFp8) {
        float svm = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((mask >> j) & 1) svm = fmaxf(svm, vs[j]);
        if (svm > vref) {
          fv = vref / svm;
          vref = svm;
          rvref = 1.f / svm;
        }
      }
      l *= fm;
      const float fo = fm * fv;
      const float mu = (m == -INFINITY) ? 0.f : m;  // masked entries are -inf and give 0
      uint32_t pk[32], pl[32];
      {
        // columns in pairs, two per packed fp32 instruction; running sums of
        // the even (ra) and odd (rb) columns in 4 chains each
        float ra[4] = {0.f, 0.f, 0.f, 0.f}, rb[4] = {0.f, 0.f, 0.f, 0.f};
        float vr[4] = {1.f, 1.f, 1.f, 1.f};
        if constexpr (Gm::kFp8) {
#pragma unroll
          for (int j = 0; j < 4; ++j) vr[j] = vs[j] * rvref;  // <= 1 up to an ulp
        }
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float ya, yb;
          fma2(ya, yb, xs[c], xs[c + 1], cj[c >> 4], cj[c >> 4], -mu, -mu);
          const float pa = ex2(ya), pb = ex2(yb);
          const int i = (c >> 1) & 3;
          add2(ra[i], rb[i], ra[i], rb[i], pa, pb);
          float wa = pa, wb = pb;
          if constexpr (Gm::kFp8) mul2(wa, wb, pa, pb, vr[c >> 4], vr[c >> 4]);
          pk[c >> 1] = pack_f32x2(wa, wb, kBfMma);
          if constexpr (Gm::kSplitP) {
            float da, db;
            sub2(da, db, wa, wb, unpack_lo(pk[c >> 1], kBfMma), unpack_hi(pk[c >> 1], kBfMma));
            pl[c >> 1] = pack_f32x2(da, db, kBfMma);
          }
        }
        l += ((ra[0] + ra[1]) + (ra[2] + ra[3])) + ((rb[0] + rb[1]) + (rb[2] + rb[3]));
      }


      // O is rescaled once PV(t - 1) is done, before PV(t) is issued (which
      // waits for this warp's P(t) below)
      if (t > 0 && __any_sync(kFull, fo != 1.f)) {
        ok = mbar_wait_bounded(&my_pv[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u, p.timeout_ns) && ok;
        tc::fence_after_sync();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tc::tmem_ld32(t_row + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fo);
          tc::tmem_st32(t_row + c0, o);
        }
      }
      // P row -> tensor memory over this row's S(t) (P_hi, then P_lo for bf16),
      // then this warp's share of P(t) is handed to its warpgroup's MMA warp
      if constexpr (Gm::kSplitP) {
        uint32_t pp[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          pp[i] = pk[i];
          pp[32 + i] = pl[i];
        }
        tc::tmem_st64(t_s, pp);
      } else {
        tc::tmem_st32(t_s, pk);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&my_p[t & 1]);
    }

    if (!aborted && T > 0) {
      ok = mbar_wait_bounded(&my_pv[(T - 1) & 1], (uint32_t)((T - 1) >> 1) & 1u, p.timeout_ns) && ok;
      if (leave()) aborted = true;
    }
    if (aborted) {
      if (lane == 0) {
        *abort_flag = 1;
        raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
      }
    } else {
      tc::fence_after_sync();
      const float inv = l > 0.f ? (Gm::kFp8 ? vref : 1.f) / l : 0.f;
      uint8_t* dst = reinterpret_cast<uint8_t*>(p.out) + orow * 2;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tc::tmem_ld32(t_row + c0, o);
        if (row_ok) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = pack_f32x2(__uint_as_float(o[8 * k + 2 * i]) * inv,
                                __uint_as_float(o[8 * k + 2 * i + 1]) * inv, QBF16);
            *reinterpret_cast<uint4*>(dst + (c0 + 8 * k) * 2) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (tid == (Gm::k16 ? 0 : (NWG * 4 + 1 + NWG) * 32)) {
    // tiles issued but never consumed by this thread (the first compute thread
    // for 16-bit caches, the first dequantization thread otherwise; only after
    // a timeout) land before the CTA exits
    const int issued = *n_issued_slot;
    bool drained = true;
    for (int k = n_prepared; k < issued; ++k)
      drained = mbar_wait_bounded(&bar_full[k % kStages], (uint32_t)(k / kStages) & 1u, p.drain_ns) && drained;
    if (!drained) raise_flag(p.err, PQKV_DEVERR_DRAIN);
  }
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Gm::kTmemCols);
  }
}

// ---- launch ------------------------------------------------------------------

template <int KVF, int D, bool QBF16>
static cudaError_t launch_prefill_t(const CUtensorMap& tmap, const PrefillParams& p, cudaStream_t st) {
  auto kern = paged_prefill_kernel<KVF, D, QBF16>;
  constexpr int smem = PrefillGeom<KVF, D>::kSmem;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  cudaLaunchConfig_t cfg = {};
  constexpr int NWG = PrefillGeom<KVF, D>::NWG;
  cfg.gridDim = dim3((unsigned)(p.B * ((p.tiles_per_seq + NWG - 1) / NWG)), (unsigned)p.Hkv);
  cfg.blockDim = dim3(PrefillGeom<KVF, D>::kThreads);
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

size_t prefill_smem_bytes(int kv_dtype, int D) {
#define PQKV_PS(F)                                                                               \
  if (kv_dtype == F) return D == 128 ? PrefillGeom<F, 128>::kSmem : PrefillGeom<F, 64>::kSmem;
  PQKV_PS(PQKV_DTYPE_FP16)
  PQKV_PS(PQKV_DTYPE_BF16)
  PQKV_PS(PQKV_DTYPE_FP8_E4M3)
  PQKV_PS(PQKV_DTYPE_FP8_E5M2)
  PQKV_PS(PQKV_DTYPE_FP4_E2M1)
#undef PQKV_PS
  return 0;
}

cudaError_t launch_prefill(int kv_dtype, int D, bool q_bf16, const CUtensorMap& tmap16, const PrefillParams& p,
                           cudaStream_t st) {
#define PQKV_PF(KVF, DD, QB) \
  if (kv_dtype == KVF && D == DD && q_bf16 == QB) return launch_prefill_t<KVF, DD, QB>(tmap16, p, st);
  PQKV_PF(PQKV_DTYPE_FP16, 128, false)
  PQKV_PF(PQKV_DTYPE_FP16, 64, false)
  PQKV_PF(PQKV_DTYPE_BF16, 128, true)
  PQKV_PF(PQKV_DTYPE_BF16, 64, true)
  PQKV_PF(PQKV_DTYPE_FP8_E4M3, 128, true)
  PQKV_PF(PQKV_DTYPE_FP8_E4M3, 128, false)
  PQKV_PF(PQKV_DTYPE_FP8_E4M3, 64, true)
  PQKV_PF(PQKV_DTYPE_FP8_E4M3, 64, false)
  PQKV_PF(PQKV_DTYPE_FP8_E5M2, 128, true)
  PQKV_PF(PQKV_DTYPE_FP8_E5M2, 128, false)
  PQKV_PF(PQKV_DTYPE_FP8_E5M2, 64, true)
  PQKV_PF(PQKV_DTYPE_FP8_E5M2, 64, false)
  PQKV_PF(PQKV_DTYPE_FP4_E2M1, 128, true)
  PQKV_PF(PQKV_DTYPE_FP4_E2M1, 128, false)
  PQKV_PF(PQKV_DTYPE_FP4_E2M1, 64, true)
  PQKV_PF(PQKV_DTYPE_FP4_E2M1, 64, false)
#undef PQKV_PF
  return cudaErrorInvalidValue;
}

}  // namespace pqkv
