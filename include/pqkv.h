/*
 * pqkv.h -- C ABI of the paged, quantized KV-cache decode-attention library.
 *
 * The operations follow the method described on three public web pages:
 *   [P1] "vLLM 0.7 Ships Unified KV Cache Compression: 3.4x Higher Concurrency
 *        on Enterprise Clusters" (dailyaiworld.com), sections "Technical
 *        Breakdown: Dynamic Quantization with Outlier Retention" (steps 1-4) and
 *        the architecture diagram (512-token chunks, FP16 outlier buffer,
 *        Flash-Decoding kernel).
 *   [P2] "vLLM v0.7.2" field report (xonoai.com/?p=2844), section
 *        "Deconstructing the v0.7.2 Architecture" (FP8 E4M3/E5M2 KV cache,
 *        16-token blocks, page tables) and "Field Observations & Production
 *        Failure Modes" (block pool exhaustion).
 *   [P3] "vLLM" glossary (inferensys.com), entries "PagedAttention" (fixed-size
 *        blocks, logical-to-physical mapping, sharing across sequences for beam
 *        search and parallel sampling), "Continuous batching" (blocks returned
 *        to the pool), "KV cache quantization" (FP8 just-in-time quantization),
 *        "Prefix caching" and "Automatic prefix caching" (requests with a
 *        common prompt prefix reuse its KV blocks), "Preemption support"
 *        (swapping KV cache blocks out to CPU RAM), "CPU offloading" and
 *        "Chunked prefill" (long prompts processed in chunks) and "Speculative
 *        decoding" (the target model verifies several proposed tokens at once).
 * Number formats follow the public OCP 8-bit Floating Point Specification
 * (OFP8: E4M3 "fn" with max 448 and no infinities, E5M2 with max 57344) and the
 * OCP Microscaling Formats specification (E2M1: values 0, .5, 1, 1.5, 2, 3, 4, 6).
 *
 * General conventions
 *  - Every pointer argument named "device" must point to GPU memory owned by the
 *    caller; every "host" pointer to CPU memory owned by the caller. The library
 *    never allocates, frees or retains device memory.
 *  - GPU entry points are asynchronous on `stream` (a cudaStream_t, 0 = legacy
 *    default stream). A return of PQKV_OK means the work was enqueued.
 *  - Problems found on the device never trap: the offending item is skipped and
 *    a PQKV_DEVERR_* bit is ORed into the caller's device int32 *err_flag (which
 *    the caller zeroes and reads back when it synchronizes).
 *  - Integer arguments are validated on the host first; invalid ones return
 *    PQKV_ERR_ARG and launch nothing.
 *
 * Cache layout (num_blocks = nb, num_kv_heads = H, head_dim = D, block = 16):
 *  One (block, head) pair holds its K tile and then its V tile contiguously, so
 *  one gathered block of one KV head is one contiguous region of the cache.
 *   FP16 / BF16 : cache  [nb][H][2 (K,V)][16][D] 2-byte elements (bit copy of input)
 *   FP8 E4M3/E5M2: cache [nb][H][2][16][D] one code per byte
 *                 scales [nb][H][4] float32 = {scale_K, scale_V, 0, 0}
 *                 (value = decode(code) * scale; 16-byte granule per pair)
 *   FP4 E2M1    : cache  [nb][H][2][16][D/2] bytes of two E2M1 codes each
 *                 K rows: row t = token t; byte i = channel 2i (low nibble)
 *                 and channel 2i+1 (high nibble)
 *                 V rows: one byte = one channel of a token pair. Pair p = 2k
 *                 (k < 4) is tokens (2k, 2k+1), pair p = 2k+1 is tokens
 *                 (2k+8, 2k+9); the even token takes the low nibble. Row p
 *                 holds channels [0, D/2) of pair p, row 8+p channels
 *                 [D/2, D); byte b of a row = channel b (+ D/2)
 *                 scales [nb][H][2][16][D/16] unsigned E4M3 codes, one per
 *                 16 consecutive channels of one token
 *                 outliers_idx [nb][H][2][8] uint8: slots 0..3 hold the outlier
 *                 channels in ascending order, 0xFF = empty; slots 4..7 = 0xFF
 *                 outliers_val [nb][H][2][16][4] IEEE fp16, value of outlier
 *                 slot r for token offset t (+0 for empty slots)
 *                 (value = channel in slot r ? outliers_val : e2m1(code)*e4m3(scale);
 *                 an outlier channel's own code is 0)
 *  Slot s addresses token offset s % 16 of physical block s / 16.
 */
#ifndef PQKV_H
#define PQKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t-compatible handle, declared here so that this header does not
 * need the CUDA headers. */
typedef struct CUstream_st* pqkv_stream_t;

/* ---- return codes ---------------------------------------------------------- */
enum {
  PQKV_OK = 0,
  PQKV_ERR_ARG = 1,   /* null pointer, bad enum, unsupported size, small buffer */
  PQKV_ERR_OOM = 2,   /* block pool cannot satisfy an allocation (no change made) */
  PQKV_ERR_STATE = 3, /* refcount underflow / freeing or sharing a free block */
  PQKV_ERR_CUDA = 4,  /* a CUDA runtime call or launch failed */
  PQKV_ERR_SCRATCH = 5 /* the request needs more than PQKV_NOALLOC_SCRATCH_BYTES of scratch */
};

/* ---- element types ---------------------------------------------------------- */
enum {
  PQKV_DTYPE_FP16 = 0,
  PQKV_DTYPE_BF16 = 1,
  PQKV_DTYPE_FP8_E4M3 = 2,
  PQKV_DTYPE_FP8_E5M2 = 3,
  PQKV_DTYPE_FP4_E2M1 = 4
};

/* ---- device error bits (ORed into *err_flag) -------------------------------- */
enum {
  PQKV_DEVERR_SLOT = 1,      /* write: slot >= 16 * num_blocks; token skipped */
  PQKV_DEVERR_BLOCK_ID = 2,  /* decode: table entry outside [0, num_blocks); block skipped */
  PQKV_DEVERR_SEQ_LEN = 4,   /* decode: seq_len < 0 or > 16 * max_blocks_per_seq; sequence
                                skipped and its output rows written as zeros */
  PQKV_DEVERR_RUN = 8,       /* write (FP8/FP4): two adjacent tokens map to the same block
                                with non-consecutive offsets */
  PQKV_DEVERR_TIMEOUT = 16,  /* a bounded wait on an asynchronous copy gave up; the kernel's
                                remaining work for that warp is skipped (outputs it owns are
                                left unwritten) after its copies in flight have landed */
  PQKV_DEVERR_DRAIN = 32     /* after a TIMEOUT, a copy still in flight did not land within the
                                full wait limit either */
};

#define PQKV_BLOCK_SIZE 16
#define PQKV_FP4_GROUP 16
#define PQKV_FP4_OUTLIER_SLOTS 4
#define PQKV_FP4_IDX_STRIDE 8
#define PQKV_FP4_SIGMA 3.2
#define PQKV_MAX_BATCH 4096

/* Library version (major * 10000 + minor * 100 + patch). */
int pqkv_version(void);

/* Human-readable name of a PQKV_* return code. Never NULL. */
const char* pqkv_status_string(int status);

/* Limit, in nanoseconds, of each wait of the attention kernels
 * (pqkv_paged_decode_attention and its variants, pqkv_paged_prefill_attention)
 * on an asynchronous copy, on a tensor-core product or on another warp of the
 * same CTA, for the launches enqueued after this call (process-wide; 0
 * restores the default of 2 s). A wait that runs out sets PQKV_DEVERR_TIMEOUT
 * and ends that warp's work, after its copies and products still in flight
 * have completed (that wait keeps the 2 s limit; PQKV_DEVERR_DRAIN if it runs
 * out too). Meant for tests of the timeout path: a very short limit makes
 * waits give up while the work they wait for is still on the way. */
void pqkv_set_decode_wait_limit_ns(uint64_t ns);

/*
 * Byte sizes of the four cache arrays for `kv_dtype`: out_bytes[0] = cache,
 * [1] = scales, [2] = outliers_idx, [3] = outliers_val (0 where the format has
 * no such array). Layout as in the header comment. Sizing the pool is the
 * caller's decision (vLLM's --gpu-memory-utilization in [P1]/[P2] launch
 * configurations). head_dim must be 64 or 128; num_blocks, num_kv_heads >= 1.
 */
int pqkv_cache_layout(int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                      size_t out_bytes[4]);

/*
 * Quantizing cache write ([P1] steps 1-3; [P2] FP8 KV cache; [P3] "KV cache
 * quantization"). Token i (0 <= i < num_tokens) of k and v, each
 * [num_tokens][num_kv_heads][head_dim] contiguous device arrays of `in_dtype`
 * (FP16 or BF16), is stored at slot slot_mapping[i] (device int32; < 0 = skip).
 *   16-bit kv_dtype: bit copy; requires in_dtype == kv_dtype.
 *   FP8: tokens are grouped into runs (maximal chains of consecutive tokens
 *     whose slots increase by one inside one block). Per run, head and K|V:
 *     a = max |x| over the run; s_run = fp32(a / FPMAX) (448 or 57344). If the
 *     run starts at offset 0 the block scale becomes s_run; otherwise
 *     s = max(s_old, s_run) and, if it grew, the existing codes at offsets below
 *     the run are re-encoded as enc(fp32(fp32(dec(c) * s_old) / s)). New codes
 *     are enc(fp32(x / s)) (all +0 when s == 0); enc rounds to nearest even and
 *     saturates to +-FPMAX, keeping the sign of zero.
 *   FP4: for a run starting at offset 0, per head and K|V: channel norm
 *     n_c = max_t |x_tc| over the run; mu and sigma (population) of the D norms
 *     in fp64; channels with n_c >= mu + 3.2 sigma are outliers, at most 4 kept
 *     (largest n_c first, ties to the lower channel), stored ascending. Runs
 *     starting later reuse the stored set. Per token: outlier values -> fp16
 *     (round to nearest even); per 16-channel group over non-outlier channels,
 *     scale code = e4m3(fp32(absmax / 6)) and codes e2m1(fp32(x / dec(scale)))
 *     (code +0 for outlier channels and when the decoded scale is 0).
 * A block must not receive tokens from two different runs in one call, and a
 * run not starting at offset 0 must append to a block written earlier. Inputs
 * must be finite. err_flag: device int32, never NULL.
 */
int pqkv_kv_cache_write(const void* k, const void* v, int in_dtype, int num_tokens,
                        const int32_t* slot_mapping, void* cache, void* scales,
                        void* outliers_idx, void* outliers_val, int kv_dtype,
                        int num_blocks, int num_kv_heads, int head_dim,
                        int32_t* err_flag, pqkv_stream_t stream);

/*
 * Device workspace needed by pqkv_paged_decode_attention for these sizes, on
 * the current device. split_blocks as in pqkv_paged_decode_attention. Returns 0
 * for invalid sizes. num_q_heads / num_kv_heads may be up to 16 here (the
 * columns of one multi-query pass); the decode itself takes up to 8.
 */
size_t pqkv_decode_workspace_bytes(int batch, int num_q_heads, int num_kv_heads,
                                   int head_dim, int max_blocks_per_seq,
                                   int split_blocks);

/*
 * Split-K paged decode attention with log-sum-exp merge ([P1] steps 3-4 and the
 * "Flash-Decoding Kernel" of its diagram; [P3] "PagedAttention").
 * For sequence b and query head hq (kv head h = hq / (num_q_heads/num_kv_heads)):
 *   L = seq_lens[b]; token t < L lives at offset t % 16 of physical block
 *   block_tables[b * max_blocks_per_seq + t / 16];
 *   out[b][hq] = sum_t softmax_t(scale * q[b][hq] . k_t) * v_t
 * with k_t, v_t dequantized from the cache. q and out: [batch][num_q_heads]
 * [head_dim] device arrays of q_dtype (FP16 or BF16); BF16/FP16 caches need
 * q_dtype == kv_dtype. num_q_heads / num_kv_heads must be an integer 1..8.
 * Table entries at and beyond ceil(L/16) are never read; a physical block may
 * appear in several tables. L == 0 gives zero output rows.
 * split_blocks: 0 = balance the work of all sequences and heads evenly over the
 * GPU; > 0 = process the KV of all (sequence, head) pairs, laid end to end, in
 * chunks of exactly that many 16-token blocks. Results differ only by rounding.
 * workspace: device buffer of at least pqkv_decode_workspace_bytes(...) bytes,
 * scratch for the split pieces and one arrival word per chunk. One kernel runs
 * on `stream`: the split decode, whose warp that writes the last piece of a
 * pair split into at most 4 pieces merges the pieces by log-sum-exp in chunk
 * order; pairs split into more pieces (long sequences) are merged by warps of
 * the same grid after their own share of the KV. The arrival words carry a tag
 * of the launch whose top byte is 0xFF, so the buffer needs no clearing
 * between calls, also when its layout (batch, heads, q_len, blocks per
 * sequence, split) changes: zero bytes and the partial outputs of earlier
 * calls never match a tag. Other old contents (a buffer's first use) match a
 * tag with probability about 2^-40 per split pair, which
 * pqkv_decode_workspace_init (zero fill) removes. Calls that share a workspace
 * must be ordered.
 * batch <= PQKV_MAX_BATCH.
 */
int pqkv_paged_decode_attention(const void* q, int q_dtype, int batch, int num_q_heads,
                                const void* cache, const void* scales,
                                const void* outliers_idx, const void* outliers_val,
                                int kv_dtype, int num_blocks, int num_kv_heads,
                                int head_dim, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* seq_lens,
                                float scale, int split_blocks, void* out,
                                void* workspace, size_t workspace_bytes,
                                int32_t* err_flag, pqkv_stream_t stream);

/*
 * Multi-query decode for speculative verification ([P3] "Speculative
 * decoding": the target model verifies several proposed tokens in one pass).
 * Each sequence has q_len query tokens, its last q_len positions (their K/V are
 * written to the cache first and seq_lens[b] counts them): token i sits at
 * position seq_lens[b] - q_len + i and attends to positions 0..that one. q and
 * out are [batch][q_len][num_q_heads][head_dim] (device, contiguous). The
 * decode kernels take the query rows of a KV head as the columns of one or two
 * 8-column tensor-core tiles: kp = min(q_len, 16 / G) consecutive query tokens
 * (G = num_q_heads / num_kv_heads <= 8) share each read of the KV, in one tile
 * when kp x G <= 8, else two; more tokens take ceil(q_len / kp) passes, each
 * reading the KV once more (long chunks: pqkv_paged_prefill_attention).
 * 1 <= q_len <= 64. workspace: at least
 * pqkv_multi_query_decode_workspace_bytes(batch, q_len, ...) bytes. A sequence
 * with 0 < seq_lens[b] < q_len gets zero rows and PQKV_DEVERR_SEQ_LEN.
 * q_len = 1 is pqkv_paged_decode_attention, bit for bit. Other arguments,
 * results and errors as there.
 */
/* Device workspace needed by pqkv_paged_multi_query_decode_attention for these
 * sizes, on the current device: pqkv_decode_workspace_bytes with the columns of
 * one pass (num_q_heads x kp, kp as above). split_blocks as there. Returns 0 for
 * sizes the call rejects (q_len outside 1..64, more than 8 query heads per KV
 * head, the other checks of pqkv_decode_workspace_bytes) or without a device. */
size_t pqkv_multi_query_decode_workspace_bytes(int batch, int q_len, int num_q_heads,
                                               int num_kv_heads, int head_dim,
                                               int max_blocks_per_seq, int split_blocks);
int pqkv_paged_multi_query_decode_attention(const void* q, int q_dtype, int batch, int q_len,
                                            int num_q_heads, const void* cache, const void* scales,
                                            const void* outliers_idx, const void* outliers_val,
                                            int kv_dtype, int num_blocks, int num_kv_heads,
                                            int head_dim, const int32_t* block_tables,
                                            int max_blocks_per_seq, const int32_t* seq_lens,
                                            float scale, int split_blocks, void* out,
                                            void* workspace, size_t workspace_bytes,
                                            int32_t* err_flag, pqkv_stream_t stream);

/*
 * pqkv_paged_decode_attention without a workspace argument, for callers that
 * cannot allocate device memory (for example a host whose device memory is
 * fully reserved by its own pool, or a latency-critical path where cudaMalloc
 * and its possible device synchronization are not acceptable). The pages
 * describe no counterpart; this is a property of this library only.
 * The scratch is one static device array of PQKV_NOALLOC_SCRATCH_BYTES that
 * every GPU loading the library holds until exit. Requests needing more
 * (pqkv_decode_workspace_bytes of the same sizes) return PQKV_ERR_SCRATCH and
 * launch nothing; with split_blocks = 0, head_dim <= 128 and up to 8 query heads
 * per KV head the need stays below 16 MiB on a 148-SM GPU. Nothing is
 * allocated. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and should come before any stream capture; the
 * address is kept for the life of the process, so a device reset
 * (cudaDeviceReset) leaves this entry point unusable, and devices numbered 64
 * or higher get PQKV_ERR_CUDA. All calls share the array, which keeps the last
 * call's contents: calls that overlap on the GPU (other streams, other host
 * threads) race on it and must be ordered by the caller. When a call's sizes
 * (batch, head counts, head_dim, max_blocks_per_seq, split_blocks) differ from
 * the previous call's on the device, the part of the array it uses is zeroed
 * first on `stream` (a memset, no allocation), so that nothing a call with
 * another layout left there is taken for this call's split-pair bookkeeping.
 * Other arguments, results and errors (checked in the same order, before the
 * scratch limit) as pqkv_paged_decode_attention.
 */
#define PQKV_NOALLOC_SCRATCH_BYTES (16u << 20)
int pqkv_paged_decode_attention_noalloc(const void* q, int q_dtype, int batch, int num_q_heads,
                                        const void* cache, const void* scales,
                                        const void* outliers_idx, const void* outliers_val,
                                        int kv_dtype, int num_blocks, int num_kv_heads,
                                        int head_dim, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* seq_lens,
                                        float scale, int split_blocks, void* out,
                                        int32_t* err_flag, pqkv_stream_t stream);

/*
 * Chunked-prefill attention over the paged cache ([P3] "Chunked prefill": a
 * long prompt is processed in chunks; [P1] architecture diagram: 512-token
 * chunks, and step 4: the attention kernel reads the compressed codes and the
 * fp16 outlier channels together; [P3] "PagedAttention": K/V through the
 * block table). Sequence b's query tokens are rows cu_q_lens[b] ..
 * cu_q_lens[b+1]-1 of q ([cu_q_lens[batch]][num_q_heads][head_dim], device,
 * q_dtype FP16 or BF16; 16-bit caches need q_dtype == kv_dtype); they are its
 * last qn_b = cu_q_lens[b+1] - cu_q_lens[b] positions, i.e. the chunk's K/V are
 * written into the cache first (pqkv_kv_cache_write) and seq_lens[b] counts
 * them. Query token i sits at position p = seq_lens[b] - qn_b + i and attends
 * to positions 0..p (causal): out_row = softmax(scale * q K[0..p]^T) V[0..p],
 * written to the same row of out (same shape and dtype as q). Query head hq
 * reads KV head hq / (num_q_heads / num_kv_heads); that ratio must divide 128.
 * cu_q_lens: device int32 [batch + 1], non-decreasing. max_q_len (host) bounds
 * every qn_b: rows past it are not computed and PQKV_DEVERR_SEQ_LEN is set. A
 * sequence with qn_b > seq_lens[b] or seq_lens[b] > 16 * max_blocks_per_seq
 * gets zero rows and PQKV_DEVERR_SEQ_LEN; tokens of a block id outside
 * [0, num_blocks) are skipped (PQKV_DEVERR_BLOCK_ID). One kernel on `stream`,
 * on the tensor cores (tcgen05); no workspace.
 */
int pqkv_paged_prefill_attention(const void* q, int q_dtype, int batch, int max_q_len,
                                 int num_q_heads, const int32_t* cu_q_lens, const void* cache,
                                 const void* scales, const void* outliers_idx,
                                 const void* outliers_val, int kv_dtype, int num_blocks,
                                 int num_kv_heads, int head_dim, const int32_t* block_tables,
                                 int max_blocks_per_seq, const int32_t* seq_lens, float scale,
                                 void* out, int32_t* err_flag, pqkv_stream_t stream);

/*
 * Whole-block copy for copy-on-write ([P3] PagedAttention: blocks shared across
 * sequences for beam search and parallel sampling; a sequence that forks off a
 * shared partial block writes into its own copy). pairs: device int32
 * [num_pairs][2] = (src, dst) block ids. Each pair copies everything the
 * block holds for all KV heads: its K/V codes and, per format, its scales and
 * outlier buffers (for the cache arrays of the formats above; unused arrays
 * may be NULL). Destinations must be distinct and not among the sources of the
 * same call. An id outside [0, num_blocks) skips the pair and sets
 * PQKV_DEVERR_BLOCK_ID in *err_flag. One kernel on `stream`.
 */
int pqkv_copy_blocks(void* cache, void* scales, void* outliers_idx, void* outliers_val,
                     int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                     const int32_t* pairs, int num_pairs, int32_t* err_flag,
                     pqkv_stream_t stream);

/*
 * Block swap to host memory ([P3] "Preemption support": KV cache blocks are
 * swapped out to CPU RAM under memory pressure and back in later; "CPU
 * offloading"). A swapped block is one record of
 * pqkv_block_record_bytes(kv_dtype, num_kv_heads, head_dim) bytes: the block's
 * cache bytes (all heads, K and V), then its scales, outlier indices and
 * outlier values as far as the format has them, each in the cache's own layout.
 * host_records: page-locked host memory (cudaHostAlloc / cudaHostRegister) of
 * num records (record i for block_ids[i]); the GPU reads or writes it
 * directly, so no device staging buffer is needed. block_ids: device int32
 * [num]. pqkv_swap_out copies blocks into records, pqkv_swap_in records into
 * blocks (ids distinct). An id outside [0, num_blocks) skips its record and
 * sets PQKV_DEVERR_BLOCK_ID. host_records not accessible from the device ->
 * PQKV_ERR_ARG. One kernel on `stream`.
 */
size_t pqkv_block_record_bytes(int kv_dtype, int num_kv_heads, int head_dim);
int pqkv_swap_out(const void* cache, const void* scales, const void* outliers_idx,
                  const void* outliers_val, int kv_dtype, int num_blocks, int num_kv_heads,
                  int head_dim, const int32_t* block_ids, int num, void* host_records,
                  int32_t* err_flag, pqkv_stream_t stream);
int pqkv_swap_in(void* cache, void* scales, void* outliers_idx, void* outliers_val,
                 int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                 const int32_t* block_ids, int num, const void* host_records,
                 int32_t* err_flag, pqkv_stream_t stream);

/* Zero-fill a decode workspace on `stream`. Optional: it only removes the
 * chance (about 2^-40 per split pair) that a never-used buffer's arbitrary old
 * bytes match a launch tag (see pqkv_paged_decode_attention). */
int pqkv_decode_workspace_init(void* workspace, size_t workspace_bytes,
                               pqkv_stream_t stream);

/*
 * Element-wise encoder used by the cache write: n float32 values (device) to
 * codes (device, one byte each) of FP8 E4M3, FP8 E5M2 or E2M1 (low nibble),
 * round to nearest even with saturation to the largest finite value, sign of
 * zero kept. Inputs must be finite.
 */
int pqkv_encode(const float* x, int64_t n, int code_dtype, uint8_t* codes,
                pqkv_stream_t stream);

/*
 * Read-bandwidth probe (a measurement helper, not a step of the method): the
 * paged gather of pqkv_paged_decode_attention without its arithmetic. Every
 * K|V tile of every (sequence, KV head, block) that a decode of the same batch
 * reads through block_tables ([P3] "PagedAttention") is copied into shared
 * memory; one word of each is XORed into *checksum (device uint32, which the
 * caller zeroes) so that no copy can be skipped. The scales and outlier
 * buffers are not read. With an identity table (sequence b's block j stored
 * right after its block j - 1) it reads the cache front to back, the
 * contiguous read ceiling. Arguments as in pqkv_paged_decode_attention;
 * lengths outside [0, 16 * max_blocks_per_seq] count as empty and block ids
 * outside [0, num_blocks) set PQKV_DEVERR_BLOCK_ID. One kernel on `stream`.
 */
int pqkv_read_probe(const void* cache, int kv_dtype, int num_blocks, int num_kv_heads, int head_dim,
                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
                    int batch, uint32_t* checksum, int32_t* err_flag, pqkv_stream_t stream);

/* ---- block pool ([P3] PagedAttention / continuous batching; [P2] pool
 *      exhaustion) ------------------------------------------------------------
 * Host-only allocator of physical block ids 0..num_blocks-1 with reference
 * counts, so that one block can sit in several block tables. O(1) per block.
 * Not thread-safe: one scheduler thread owns a pool. */
typedef struct pqkv_pool pqkv_pool;

/* Create a pool with all blocks free. Allocation hands out the lowest free ids
 * first on a fresh pool, then reuses freed ids last-in first-out. */
int pqkv_pool_create(int32_t num_blocks, pqkv_pool** out_pool);
void pqkv_pool_destroy(pqkv_pool* pool);
/* Allocate n blocks into ids_out (host), refcount 1 each. All or nothing:
 * PQKV_ERR_OOM leaves the pool unchanged. */
int pqkv_pool_alloc(pqkv_pool* pool, int n, int32_t* ids_out);
/* Add one reference to each of ids[0..n) (host). Every id must be allocated;
 * otherwise PQKV_ERR_STATE (or ERR_ARG for an id out of range), no change. */
int pqkv_pool_share(pqkv_pool* pool, const int32_t* ids, int n);
/* Drop one reference from each of ids[0..n) (host); blocks reaching 0 return to
 * the pool. Dropping more references than an id holds (counting repeats in
 * ids) gives PQKV_ERR_STATE and no change. */
int pqkv_pool_free(pqkv_pool* pool, const int32_t* ids, int n);
/* Blocks neither referenced nor cached. */
int32_t pqkv_pool_num_free(const pqkv_pool* pool);
/* Reference count of `id`, or -1 if out of range. */
int32_t pqkv_pool_refcount(const pqkv_pool* pool, int32_t id);

/*
 * Prefix cache ([P3] "Prefix caching", "Automatic prefix caching"). Only full
 * 16-token blocks are cached. A cached block is identified by its 16 token ids
 * and by the cache entry of the block before it in the prompt, so a hit always
 * means the same whole prefix (no hashing shortcut can return another
 * prefix's block). A cached block that no sequence references stays cached and
 * is "evictable": pqkv_pool_alloc / pqkv_pool_cow take free blocks first, then
 * evict the least recently released evictable block (dropping its entry; the
 * entries that continued its prefix can then never be found again and are
 * evicted in their turn). Cached blocks must not be written: a sequence that
 * appends into a block it shares, or into a cached block, calls pqkv_pool_cow
 * first.
 */
int32_t pqkv_pool_num_evictable(const pqkv_pool* pool);
/* Number of cache entries (referenced or evictable). */
int32_t pqkv_pool_num_cached(const pqkv_pool* pool);
/* Longest cached prefix of token_ids[0..num_tokens) (host), in whole blocks:
 * writes the ids of the hit blocks to ids_out (host, room for num_tokens/16)
 * and their count to *num_hit; each hit block gains one reference (an evictable
 * one stops being evictable). A caller that must compute at least one token
 * passes num_tokens = prompt length - 1. */
int pqkv_pool_prefix_lookup(pqkv_pool* pool, const int32_t* token_ids, int num_tokens,
                            int32_t* ids_out, int* num_hit);
/* Register the full blocks of a prompt whose KV has been written: block b of
 * token_ids[0..num_tokens) lives in ids[b] (host, b < min(num_tokens/16,
 * num_ids); every id referenced). Blocks whose prefix is cached already (in
 * that block, as returned by a lookup, or in another one) are skipped. From the
 * first prefix not cached on, each block becomes a new entry; such a block
 * already cached under another prefix, or repeated, gives PQKV_ERR_STATE and no
 * change. References are not changed. */
int pqkv_pool_prefix_insert(pqkv_pool* pool, const int32_t* token_ids, int num_tokens,
                            const int32_t* ids, int num_ids);
/* Copy-on-write before writing into block `id` (referenced by the caller).
 * If the caller holds the only reference and the block is not cached, *new_id
 * = id and *copy_needed = 0. Otherwise a block is allocated (as
 * pqkv_pool_alloc), the caller's reference moves from `id` to it, *new_id is
 * that block and *copy_needed = 1: the caller then copies `id` into it with
 * pqkv_copy_blocks before writing. PQKV_ERR_OOM / ERR_STATE: no change. */
int pqkv_pool_cow(pqkv_pool* pool, int32_t id, int32_t* new_id, int* copy_needed);

/*
 * Host helper: slot mapping for appending tokens. For each sequence b, tokens
 * at positions start_pos[b] .. start_pos[b] + num_new[b] - 1 get
 * slot = block_tables[b][pos / 16] * 16 + pos % 16, written consecutively into
 * slots_out (host int32, sum(num_new) entries). Returns PQKV_ERR_ARG if a
 * position needs a table entry outside [0, max_blocks_per_seq) or a negative id.
 */
int pqkv_build_slot_mapping(const int32_t* block_tables, int batch,
                            int max_blocks_per_seq, const int32_t* start_pos,
                            const int32_t* num_new, int32_t* slots_out);

#ifdef __cplusplus
}
#endif
#endif /* PQKV_H */
