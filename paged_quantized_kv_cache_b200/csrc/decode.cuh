// decode.cuh -- split-K paged decode attention with in-register dequantization
// and log-sum-exp merge, for sm_100a.
//
// Method ("vLLM 0.7 Ships Unified KV Cache Compression": architecture diagram
// "Flash-Decoding Kernel" and step 4, "Flash-Decoding kernels fuse the outlier
// and compressed representations"; "vLLM" glossary, "PagedAttention"):
// every (sequence, KV head) pair reads its KV blocks through the block table,
// the KV range is split across the GPU, each piece keeps an online softmax
// (running max m, sum l, unnormalized output O) and the pieces of one pair are
// merged by log-sum-exp.
//
// Work decomposition. The blocks of all (sequence b, KV head h) pairs are laid
// end to end (b-major, then h, then block j) into one flat range of T blocks.
// The grid is persistent (one CTA per SM, NW warps each); the flat range is cut
// into W equal shares, one per warp (W = all warps), and a fixed split also cuts
// it at every multiple of split_blocks (SplitPlan); the cells are the units.
// A unit covers whole pairs (written straight to `out`) and at most two
// partial pairs at its ends (written to a workspace slot). The pieces of a
// split pair are merged in unit order, so results do not depend on timing:
// a pair of at most kMergeInKernel pieces (the usual case: many sequences)
// by the warp that writes its last piece (counted in a per-pair arrival
// word); a longer one (few long sequences spread over the GPU) column by
// column, each column by one warp of the same grid once its own share is
// done, when the arrival word shows all pieces.
//
// Per warp: a private ring of NS shared-memory stages, each holding the K and V
// tiles of one (block, head) pair fetched by one TMA tensor copy (128/64/32-byte
// swizzle so ldmatrix reads are conflict-free) plus small bulk copies of the
// block's scales and outlier buffer. Lane 0 issues the copies NS blocks ahead.
// GQA: the G = Hq/Hkv query heads of a KV head are the N = 8 columns of
// m16n8k16 MMAs: S^T = K Q^T (M = 16 tokens of one block) and O^T += V^T P^T
// (M = 16 head dims per tile, K = 16 tokens). Dequantization happens in
// registers between ldmatrix and the MMA.
#pragma once

#include "common.cuh"

namespace pqkv {

constexpr int kDecodeWarps = 12;  // upper bound of warps per CTA over all formats
constexpr int kMergeInKernel = 4;  // split pairs of up to this many pieces are merged inside the decode

struct DecodeParams {
  const void* q;
  void* out;
  const uint8_t* scales;        // FP8: float [nb][H][4]; FP4: u8 [nb][H][2][16][D/16]
  const uint8_t* oidx;          // FP4: u8 [nb][H][2][8]
  const uint8_t* oval;          // FP4: fp16 [nb][H][2][16][4]
  const int32_t* block_tables;  // [B][maxblk]
  const int32_t* seq_lens;      // [B]
  int32_t* err;
  float* partials;              // [2 * chunks][slot_floats]
  unsigned long long* counters; // [chunks] arrival words of split pairs (tag << 24 | pieces)
  // G = MMA columns per KV head = Gh query heads x the query tokens q0,
  // q0 + 1, ... of this pass (column c = token q0 + c / Gh, head c % Gh); k > 1
  // is multi-query decode: token i of a sequence of length L sits at position
  // L - k + i and sees positions <= it
  int B, Hq, Hkv, G, nb, maxblk;
  int k, Gh, q0;
  int split_blocks;
  int slot_floats;
  float scale_log2;             // softmax scale * log2(e)
  uint64_t timeout_ns;          // limit of a wait on a copy before the warp gives up
  uint64_t drain_ns;            // after giving up: limit of the wait for copies still in flight
  unsigned long long epoch;     // tag of this launch (40 bits, never 0)
};

// The split of the flat block range (T blocks of all (sequence, head) pairs,
// laid end to end) over the W warps of the decode grid: warp w takes blocks
// [w Qw, (w + 1) Qw), Qw = ceil(T / W), so every warp has the same share. With
// a fixed split (split_blocks = C > 0) a piece of a pair also ends at every
// multiple of C, so that each partial result lies inside one C-block chunk of
// the split; the balanced split has C = Qw. The cells between consecutive
// boundaries (multiples of Qw or of C) are the units; a pair's pieces are the
// units its blocks cross, in order, and a piece's workspace slot is indexed by
// its unit (there are at most ceil(T / C) + W of them).
struct SplitPlan {
  int Qw, C;
  long long lcm;  // of Qw and C: boundaries that are both count once
  __device__ __forceinline__ int unit(int f) const {  // the unit holding flat block f
    return f / C + f / Qw - (int)((long long)f / lcm);
  }
};

__device__ __forceinline__ SplitPlan make_split_plan(int T, int W, int split_blocks) {
  SplitPlan s;
  s.Qw = max(1, (T + W - 1) / W);
  s.C = split_blocks > 0 ? split_blocks : s.Qw;
  int a = s.Qw, b = s.C;
  while (b != 0) {
    const int t = a % b;
    a = b;
    b = t;
  }
  s.lcm = (long long)(s.Qw / a) * s.C;
  return s;
}

// Compile-time geometry of one format; NT = tiles of 8 MMA columns (query rows)
// per KV head: 1, or 2 for multi-query decode with up to 16 rows.
template <int KVF, int D, int NT = 1>
struct DecodeGeom {
  static constexpr bool k16 = (KVF == PQKV_DTYPE_FP16 || KVF == PQKV_DTYPE_BF16);
  static constexpr bool kFp8 = (KVF == PQKV_DTYPE_FP8_E4M3 || KVF == PQKV_DTYPE_FP8_E5M2);
  static constexpr bool kFp4 = (KVF == PQKV_DTYPE_FP4_E2M1);
  static constexpr int kRow = row_bytes(KVF, D);               // bytes per token row
  static constexpr int kBoxRow = kRow > 128 ? 128 : kRow;       // bytes per TMA box row
  static constexpr int kBoxes = kRow / kBoxRow;                 // TMA boxes per tile
  static constexpr int kTile = 32 * kRow;                       // K (16 rows) + V (16 rows)
  static constexpr int kScaleBytes = kFp8 ? 16 : (kFp4 ? 2 * 16 * (D / 16) : 0);
  static constexpr int kValBytes = kFp4 ? 2 * 16 * 4 * 2 : 0;
  static constexpr int kIdxBytes = kFp4 ? 16 : 0;
  static constexpr int kSide = kScaleBytes + kValBytes + kIdxBytes;  // multiple of 16
  static constexpr int kSideStride = kSide == 0 ? 0 : ((kSide + 127) / 128) * 128;
  // Warps per CTA and shared-memory stages per warp; about 192-200 KB of stages
  // per SM. Blocks are consumed two at a time, so while a pair is computed NS - 2
  // copies stay in flight: 16-bit D128 with one column tile takes 5 warps x 5
  // stages (measured 1.2% faster per step than 6 x 4 on the llama8b workload);
  // with two tiles the longer compute per block favours 6 x 4 (q_len 4: 4865
  // against 4507 GB/s). Two tiles double the accumulators: quantized formats
  // then drop to 8 warps.
  static constexpr int kWarps = k16 ? (D == 128 ? (NT == 1 ? 5 : 6) : 8) : (NT == 1 ? 12 : 8);
  static constexpr int kCols = 8 * NT;                          // MMA columns per KV head
  static constexpr int kStages = k16 ? (D == 128 ? (NT == 1 ? 5 : 4) : 6) : (D == 128 ? 4 : 6);
  static constexpr uint32_t kTx = kTile + kSide;
  // FP4 per-warp shared rows, padded so that the 8 rows fall in different banks
  static constexpr int kQStride = D + 2;  // f16 query copy, halves per row
  static constexpr int kOStride = D + 1;  // outlier-channel O, floats per row
  // byte offset in a tile of (row r, byte b of that row); rows 0-15 K, 16-31 V.
  __device__ static __forceinline__ uint32_t off(int r, int b) {
    const int box = b / kBoxRow;
    const int inner = b % kBoxRow;
    int chunk = inner >> 4;
    if constexpr (kBoxRow == 128) chunk ^= (r & 7);
    else if constexpr (kBoxRow == 64) chunk ^= ((r >> 1) & 3);
    else chunk ^= ((r >> 2) & 1);
    return (uint32_t)(box * 32 * kBoxRow + r * kBoxRow + (chunk << 4) + (inner & 15));
  }
};

template <int KVF, int D, int NT = 1>
struct DecodeSmem {
  using Gm = DecodeGeom<KVF, D, NT>;
  static constexpr int kTilesBytes = Gm::kWarps * Gm::kStages * Gm::kTile;
  static constexpr int kSideBytes = Gm::kWarps * Gm::kStages * Gm::kSideStride;
  static constexpr int kBarBytes = Gm::kWarps * Gm::kStages * 8;
  static constexpr int kQBytes = Gm::kFp4 ? Gm::kWarps * Gm::kCols * Gm::kQStride * 2 : 0;     // per-warp f16 q copy
  static constexpr int kOextBytes = Gm::kFp4 ? Gm::kWarps * Gm::kCols * Gm::kOStride * 4 : 0;  // outlier-channel O
  static size_t bytes(int B) {
    return 1024 + (size_t)kTilesBytes + kSideBytes + kBarBytes + kQBytes + kOextBytes + (size_t)(B + 1) * 4;
  }
};

}  // namespace pqkv
