// probe.cu -- read-bandwidth probe: the decode's paged gather without its math.
//
// It measures what the decode kernel could reach if its per-block arithmetic
// cost nothing: every (sequence, KV head, block) K|V tile that a decode of the
// same batch reads ("vLLM" glossary, "PagedAttention": logical block ->
// physical block through the block table) is pulled into shared memory by a
// bulk copy, and one word of it is folded into a checksum so that no copy can
// be dropped. Given an identity block table (block j of every sequence stored
// right after block j - 1), the same kernel reads the cache front to back,
// which gives the contiguous read ceiling beside the gathered one.
//
// Decomposition as in the decode: the tiles of all (sequence, head) pairs are
// laid end to end into one flat range; each warp of a persistent grid (one CTA
// per SM) takes one contiguous chunk of it. Lane 0 of every warp keeps a ring
// of stages in flight on its own mbarriers; all waits are bounded.
#include "common.cuh"

namespace pqkv {

namespace {

constexpr int kProbeWarps = 6;
constexpr int kProbeRingBytes = 32 * 1024;  // per warp: 4 x 8 KB (bf16 D128) .. 16 x 2 KB (FP4 D128)
constexpr int kProbeMaxStages = 16;

struct ProbeParams {
  const uint8_t* cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  uint32_t* checksum;
  int32_t* err;
  int B, Hkv, nb, maxblk;
  int tile_bytes;  // K|V bytes of one (block, head) pair
  int stages;      // ring stages per warp (tile_bytes * stages <= kProbeRingBytes)
  uint64_t timeout_ns;
  uint64_t drain_ns;
};

__global__ void __launch_bounds__(kProbeWarps * 32, 1) read_probe_kernel(const ProbeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint8_t* ring = smem + 1024;
  int* P = reinterpret_cast<int*>(ring + kProbeWarps * kProbeRingBytes);  // [B + 1]
  __shared__ int warp_sums[kProbeWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int B = p.B;
  // prefix sums of blocks per sequence (lengths outside [0, 16 * maxblk] count 0)
  {
    const int per = (B + blockDim.x - 1) / blockDim.x;
    const int lo = min(B, tid * per), hi = min(B, lo + per);
    const int lim = kBlock * p.maxblk;
    int local = 0;
    for (int i = lo; i < hi; ++i) {
      const int L = p.seq_lens[i];
      local += (L < 0 || L > lim) ? 0 : (L + kBlock - 1) / kBlock;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < warp; ++w) run += warp_sums[w];
    if (tid == 0) P[0] = 0;
    for (int i = lo; i < hi; ++i) {
      const int L = p.seq_lens[i];
      run += (L < 0 || L > lim) ? 0 : (L + kBlock - 1) / kBlock;
      P[i + 1] = run;
    }
  }
  __syncthreads();
  if (lane != 0) return;

  uint64_t* wbar = bars + warp * kProbeMaxStages;
  uint8_t* wring = ring + warp * kProbeRingBytes;
  const int NS = p.stages;
  for (int s = 0; s < NS; ++s) mbar_init(&wbar[s], 1);
  fence_mbar_init();

  const long long T = (long long)p.Hkv * P[B];
  const long long W = (long long)gridDim.x * kProbeWarps;
  const long long Q = (T + W - 1) / W;
  const long long w = (long long)warp * gridDim.x + blockIdx.x;
  const long long f0 = min(T, w * Q), f1 = min(T, f0 + Q);

  // flat tile index -> address of its K|V tile, or nullptr for a bad block id
  auto tile_at = [&](long long f) -> const uint8_t* {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if ((long long)p.Hkv * P[mid] <= f) lo = mid; else hi = mid;
    }
    const int n = P[lo + 1] - P[lo];
    const long long rel = f - (long long)p.Hkv * P[lo];
    const int h = (int)(rel / n), j = (int)(rel - (long long)h * n);
    const int id = p.block_tables[(size_t)lo * p.maxblk + j];
    if (id < 0 || id >= p.nb) return nullptr;
    return p.cache + ((size_t)id * p.Hkv + h) * (size_t)p.tile_bytes;
  };

  uint32_t phase = 0, inflight = 0, skip = 0, sum = 0;
  auto issue = [&](int s, long long f) {
    const uint8_t* src = tile_at(f);
    if (!src) {
      raise_flag(p.err, PQKV_DEVERR_BLOCK_ID);
      skip |= 1u << s;
      mbar_arrive(&wbar[s]);
    } else {
      skip &= ~(1u << s);
      mbar_arrive_expect_tx(&wbar[s], (uint32_t)p.tile_bytes);
      bulk_load(wring + s * p.tile_bytes, src, (uint32_t)p.tile_bytes, &wbar[s]);
    }
    inflight |= 1u << s;
  };
  for (int s = 0; s < NS && f0 + s < f1; ++s) issue(s, f0 + s);
  int s = 0;
  bool aborted = false;
  for (long long f = f0; f < f1; ++f) {
    if (!mbar_wait_bounded(&wbar[s], (phase >> s) & 1u, p.timeout_ns)) {  // the stage stays in flight
      raise_flag(p.err, PQKV_DEVERR_TIMEOUT);
      aborted = true;
      break;
    }
    phase ^= 1u << s;
    inflight &= ~(1u << s);
    if (!((skip >> s) & 1u))
      sum ^= *reinterpret_cast<const volatile uint32_t*>(wring + s * p.tile_bytes + (f & 7) * 16);
    if (f + NS < f1) issue(s, f + NS);
    s = (s + 1 == NS) ? 0 : s + 1;
  }
  if (aborted) {  // let the copies still in flight land before the warp exits (full limit)
    bool drained = true;
    for (int s2 = 0; s2 < NS; ++s2)
      if ((inflight >> s2) & 1u) drained = mbar_wait_bounded(&wbar[s2], (phase >> s2) & 1u, p.drain_ns) && drained;
    if (!drained) raise_flag(p.err, PQKV_DEVERR_DRAIN);
  }
  atomicXor(p.checksum, sum);
}

}  // namespace

size_t read_probe_smem_bytes(int B) { return 128 + 1024 + (size_t)kProbeWarps * kProbeRingBytes + (size_t)(B + 1) * 4; }

cudaError_t launch_read_probe(const uint8_t* cache, int kv_dtype, int nb, int H, int D, const int32_t* block_tables,
                              int maxblk, const int32_t* seq_lens, int B, uint32_t* checksum, int32_t* err,
                              uint64_t timeout_ns, int sms, cudaStream_t st) {
  ProbeParams p;
  p.cache = cache;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.checksum = checksum;
  p.err = err;
  p.B = B;
  p.Hkv = H;
  p.nb = nb;
  p.maxblk = maxblk;
  p.tile_bytes = 2 * kBlock * row_bytes(kv_dtype, D);
  p.stages = kProbeRingBytes / p.tile_bytes;
  if (p.stages > kProbeMaxStages) p.stages = kProbeMaxStages;
  p.timeout_ns = timeout_ns;
  p.drain_ns = timeout_ns;
  const size_t smem = read_probe_smem_bytes(B);
  cudaError_t e = cudaFuncSetAttribute(read_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  read_probe_kernel<<<sms, kProbeWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace pqkv
