"""Seeded synthetic inputs for the five decode workloads.

This module only draws random numbers and lays out block tables and slot
mappings; it holds none of the cache's quantization or attention arithmetic.
Both the GPU library's tests/benchmark and the CPU oracle consume what it makes.

Workloads (the pages' shapes: 16-token blocks, GQA, 512-token chunks):
  tiny    4 seqs, lens {17,33,64,100}, 8 q / 2 kv heads, D 64, fp16 KV; tables are
          one random permutation of a 64-block pool assigned in logical order.
  llama8b 64 seqs, lens U[512,4096], 32 q / 8 kv heads, D 128, bf16 KV, ids sampled
          without replacement from a 40,000-block pool.
  fp8     128 seqs, lens U[1024,8192], same heads, FP8 (E4M3 or E5M2) KV; prefill
          in one write per sequence, then one appended token per sequence.
  llama70b 16 seqs, lens U[24576,40960], 64 q / 8 kv heads, D 128, bf16 or FP8;
          sequences 0-3 share one 4096-token (256-block) prefix.
  fp4     256 seqs, lens round(exp(U(ln 1024, ln 65536))), 32 q / 8 kv heads, D 128,
          FP4 KV; two channels per (head, K|V) scaled x16; written in 512-token
          chunks across all sequences.
Every sequence draws its K/V from its own child stream of
numpy.random.SeedSequence(workload seed), so any subset can be regenerated.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, List, Optional, Sequence, Tuple

import numpy as np
import torch

BLOCK = 16

DT_FP16, DT_BF16, DT_FP8_E4M3, DT_FP8_E5M2, DT_FP4 = 0, 1, 2, 3, 4
TORCH_DTYPE = {DT_FP16: torch.float16, DT_BF16: torch.bfloat16}


@dataclasses.dataclass
class Spec:
    name: str
    seed: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_dtype: int
    q_dtype: int
    lens: str                      # "fixed" | "uniform" | "loguniform"
    len_lo: int
    len_hi: int
    fixed_lens: Optional[Sequence[int]] = None
    pool_blocks: int = 0
    append_tokens: int = 0         # tokens written per sequence after the prefill
    shared_prefix_seqs: int = 0    # sequences 0..n-1 share a prefix
    shared_prefix_tokens: int = 0
    outlier_channels: int = 0      # channels per (head, K|V) scaled by outlier_gain
    outlier_gain: float = 16.0
    chunk_tokens: int = 0          # >0: prefill written in chunks of this many tokens
    split_blocks: int = 0          # split size the workload names (0 = balanced)
    permute_pool: bool = False     # ids = permutation of the pool in logical order


def spec(name: str, kv_dtype: Optional[int] = None, batch: Optional[int] = None) -> Spec:
    """Return the workload `name`, optionally with another KV dtype or a batch cut."""
    if name == "tiny":
        s = Spec("tiny", 1, 4, 8, 2, 64, DT_FP16, DT_FP16, "fixed", 17, 100,
                 fixed_lens=(17, 33, 64, 100), pool_blocks=64, permute_pool=True)
    elif name == "llama8b":
        s = Spec("llama8b", 2, 64, 32, 8, 128, DT_BF16, DT_BF16, "uniform", 512, 4096,
                 pool_blocks=40000)
    elif name == "fp8":
        s = Spec("fp8", 3, 128, 32, 8, 128, DT_FP8_E4M3, DT_BF16, "uniform", 1024, 8192,
                 pool_blocks=65664, append_tokens=1)
    elif name == "llama70b":
        s = Spec("llama70b", 4, 16, 64, 8, 128, DT_BF16, DT_BF16, "uniform", 24576, 40960,
                 pool_blocks=40960, shared_prefix_seqs=4, shared_prefix_tokens=4096,
                 split_blocks=32)
    elif name == "fp4":
        s = Spec("fp4", 5, 256, 32, 8, 128, DT_FP4, DT_BF16, "loguniform", 1024, 65536,
                 pool_blocks=1048576, outlier_channels=2, chunk_tokens=512)
    elif name == "prefill":
        # chunked prefill: a cached prefix of U[0, 7680] tokens (written in
        # 512-token chunks) and one more 512-token chunk whose queries attend
        s = Spec("prefill", 6, 16, 32, 8, 128, DT_BF16, DT_BF16, "uniform", 0, 7680,
                 pool_blocks=9000, append_tokens=512, chunk_tokens=512)
    else:
        raise KeyError(name)
    if kv_dtype is not None:
        s.kv_dtype = kv_dtype
    if batch is not None:
        s.batch = batch
    return s


def _streams(s: Spec) -> List[np.random.SeedSequence]:
    # children 0..B-1: per-sequence K/V; B: lengths; B+1: physical ids; B+2: q;
    # B+3: shared prefix K/V; B+4: outlier channel choice; B+5: multi-token q;
    # B+6: stand-alone write-call inputs (write_kv). The number of children
    # depends only on the full batch of the named workload so that a batch cut
    # keeps every sequence's stream (a child's stream depends on its index only).
    full = spec(s.name).batch
    return np.random.SeedSequence(s.seed).spawn(full + 7)


def seq_lens(s: Spec) -> np.ndarray:
    """Context lengths of the prefill (before any appended tokens)."""
    full = spec(s.name).batch
    if s.lens == "fixed":
        out = np.array(s.fixed_lens, dtype=np.int64)
    else:
        rng = np.random.Generator(np.random.PCG64(_streams(s)[full]))
        if s.lens == "uniform":
            out = rng.integers(s.len_lo, s.len_hi, size=full, endpoint=True)
        else:
            u = rng.uniform(math.log(s.len_lo), math.log(s.len_hi), size=full)
            out = np.rint(np.exp(u)).astype(np.int64)
    return out[: s.batch].astype(np.int32)


def nblocks(n_tokens: int) -> int:
    return (n_tokens + BLOCK - 1) // BLOCK


@dataclasses.dataclass
class Tables:
    block_tables: np.ndarray       # int32 [B][max_blocks], -1 beyond a sequence's blocks
    max_blocks: int
    num_blocks: int                # pool size


def tables(s: Spec) -> Tables:
    """Physical block ids for every sequence's final length (prefill + appends)."""
    full = spec(s.name).batch
    lens = seq_lens(s) + s.append_tokens
    nb = [nblocks(int(n)) for n in lens]
    max_blocks = nblocks(max(int(spec(s.name).len_hi) + s.append_tokens, int(max(lens))))
    shared = nblocks(s.shared_prefix_tokens) if s.shared_prefix_seqs else 0
    n_share = min(s.shared_prefix_seqs, s.batch)
    need = sum(nb) - shared * max(0, n_share - 1)
    if need > s.pool_blocks:
        raise ValueError("pool too small for this workload")
    rng = np.random.Generator(np.random.PCG64(_streams(s)[full + 1]))
    if s.permute_pool:
        ids = rng.permutation(s.pool_blocks)[:need]
    else:
        ids = rng.choice(s.pool_blocks, size=need, replace=False)
    bt = np.full((s.batch, max_blocks), -1, dtype=np.int32)
    pos = 0
    prefix_ids = None
    for b in range(s.batch):
        if b < n_share and shared:
            if prefix_ids is None:
                prefix_ids = ids[pos:pos + shared]
                pos += shared
            bt[b, :shared] = prefix_ids
            rest = nb[b] - shared
            bt[b, shared:nb[b]] = ids[pos:pos + rest]
            pos += rest
        else:
            bt[b, :nb[b]] = ids[pos:pos + nb[b]]
            pos += nb[b]
    assert pos == need
    return Tables(bt, max_blocks, s.pool_blocks)


def outlier_channels(s: Spec) -> np.ndarray:
    """int64 [Hkv][2][n]: channels scaled by outlier_gain per (head, K|V)."""
    full = spec(s.name).batch
    rng = np.random.Generator(np.random.PCG64(_streams(s)[full + 4]))
    out = np.zeros((s.num_kv_heads, 2, s.outlier_channels), dtype=np.int64)
    for h in range(s.num_kv_heads):
        for kv in range(2):
            out[h, kv] = np.sort(rng.choice(s.head_dim, size=s.outlier_channels, replace=False))
    return out


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def seq_kv(s: Spec, b: int, with_append: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V of sequence b: [L(+append)][Hkv][D] in the input dtype (CPU).

    Values are N(0,1) float32 rounded to the input dtype; channels chosen by
    outlier_channels() are multiplied by outlier_gain before rounding. A shared
    prefix comes from its own stream, identical for sequences 0..n-1.
    """
    full = spec(s.name).batch
    L = int(seq_lens(s)[b]) + (s.append_tokens if with_append else 0)
    st = _streams(s)
    rng = np.random.Generator(np.random.PCG64(st[b]))
    H, D = s.num_kv_heads, s.head_dim
    start = 0
    parts_k, parts_v = [], []
    if s.shared_prefix_seqs and b < s.shared_prefix_seqs:
        prng = np.random.Generator(np.random.PCG64(st[full + 3]))
        P = s.shared_prefix_tokens
        parts_k.append(_normal(prng, (P, H, D)))
        parts_v.append(_normal(prng, (P, H, D)))
        start = P
    L0 = int(seq_lens(s)[b])
    parts_k.append(_normal(rng, (L0 - start, H, D)))
    parts_v.append(_normal(rng, (L0 - start, H, D)))
    if L > L0:
        parts_k.append(_normal(rng, (L - L0, H, D)))
        parts_v.append(_normal(rng, (L - L0, H, D)))
    k = np.concatenate(parts_k, axis=0)
    v = np.concatenate(parts_v, axis=0)
    if s.outlier_channels:
        ch = outlier_channels(s)
        for h in range(H):
            k[:, h, ch[h, 0]] *= s.outlier_gain
            v[:, h, ch[h, 1]] *= s.outlier_gain
    in_dt = torch.float16 if s.kv_dtype == DT_FP16 else (
        torch.float16 if s.q_dtype == DT_FP16 else torch.bfloat16)
    return torch.from_numpy(k).to(in_dt), torch.from_numpy(v).to(in_dt)


def write_kv(s: Spec, b: int, start: int, n: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V [n][Hkv][D] for positions start..start+n-1 of sequence b, for
    timing a write call on its own: N(0,1) with the workload's planted outlier
    channels, rounded to the input dtype, like seq_kv, but drawn from a stream
    of their own (per sequence and start) so that no sequence's full stream is
    needed. Not the values seq_kv gives for those positions."""
    full = spec(s.name).batch
    ss = np.random.SeedSequence(entropy=s.seed, spawn_key=_streams(s)[full + 6].spawn_key + (b, start))
    rng = np.random.Generator(np.random.PCG64(ss))
    H, D = s.num_kv_heads, s.head_dim
    k = _normal(rng, (n, H, D))
    v = _normal(rng, (n, H, D))
    if s.outlier_channels:
        ch = outlier_channels(s)
        for h in range(H):
            k[:, h, ch[h, 0]] *= s.outlier_gain
            v[:, h, ch[h, 1]] *= s.outlier_gain
    in_dt = TORCH_DTYPE[input_dtype(s)]
    return torch.from_numpy(k).to(in_dt), torch.from_numpy(v).to(in_dt)


def input_dtype(s: Spec) -> int:
    """dtype of the K/V fed to the cache write."""
    if s.kv_dtype in (DT_FP16, DT_BF16):
        return s.kv_dtype
    return s.q_dtype


def multi_query(s: Spec, q_len: int) -> torch.Tensor:
    """q [B][q_len][Hq][D] ~ N(0,1) rounded to the query dtype (CPU), for the
    multi-query (speculative verification) step; its own stream."""
    full = spec(s.name).batch
    rng = np.random.Generator(np.random.PCG64(_streams(s)[full + 5]))
    q = _normal(rng, (full, q_len, s.num_q_heads, s.head_dim))[: s.batch]
    return torch.from_numpy(np.ascontiguousarray(q)).to(TORCH_DTYPE[s.q_dtype])


def query(s: Spec) -> torch.Tensor:
    """q [B][Hq][D] ~ N(0,1) rounded to the query dtype (CPU)."""
    full = spec(s.name).batch
    rng = np.random.Generator(np.random.PCG64(_streams(s)[full + 2]))
    q = _normal(rng, (full, s.num_q_heads, s.head_dim))[: s.batch]
    return torch.from_numpy(np.ascontiguousarray(q)).to(TORCH_DTYPE[s.q_dtype])


def slots_for(bt_row: np.ndarray, start: int, n: int) -> np.ndarray:
    """Slots of positions start..start+n-1 of one sequence: id*16 + pos%16."""
    pos = np.arange(start, start + n, dtype=np.int64)
    return (bt_row[pos // BLOCK].astype(np.int64) * BLOCK + pos % BLOCK).astype(np.int32)


@dataclasses.dataclass
class WriteCall:
    """One cache-write call: token rows (seq, first position, count) in order."""
    rows: List[Tuple[int, int, int]]


def prefill_calls(s: Spec) -> List[WriteCall]:
    """The write calls that store every sequence's prefill.

    One call per sequence, or, with chunk_tokens, call j holds positions
    [j*chunk, (j+1)*chunk) of every sequence long enough (sequence order).
    Sequences 1..n-1 of a shared prefix skip the prefix: sequence 0 wrote it.
    """
    lens = seq_lens(s)
    first = np.zeros(s.batch, dtype=np.int64)
    if s.shared_prefix_seqs:
        first[1:min(s.shared_prefix_seqs, s.batch)] = s.shared_prefix_tokens
    calls: List[WriteCall] = []
    if s.chunk_tokens:
        c = s.chunk_tokens
        nchunks = (int(lens.max()) + c - 1) // c
        for j in range(nchunks):
            rows = []
            for b in range(s.batch):
                lo = max(j * c, int(first[b]))
                hi = min((j + 1) * c, int(lens[b]))
                if hi > lo:
                    rows.append((b, lo, hi - lo))
            if rows:
                calls.append(WriteCall(rows))
    else:
        for b in range(s.batch):
            if int(lens[b]) > int(first[b]):
                calls.append(WriteCall([(b, int(first[b]), int(lens[b]) - int(first[b]))]))
    return calls


def append_call(s: Spec) -> Optional[WriteCall]:
    """The decode-step write: append_tokens new tokens per sequence."""
    if not s.append_tokens:
        return None
    lens = seq_lens(s)
    return WriteCall([(b, int(lens[b]), s.append_tokens) for b in range(s.batch)])


def gather_call(s: Spec, call: WriteCall, tab: Tables, kv_cache=None):
    """Materialize a write call: (k, v, slots) CPU tensors / int32 array.

    kv_cache: optional dict b -> (k, v) from seq_kv() to avoid regenerating.
    """
    ks, vs, sl = [], [], []
    for (b, lo, n) in call.rows:
        if kv_cache is not None and b in kv_cache:
            k, v = kv_cache[b]
        else:
            k, v = seq_kv(s, b)
        ks.append(k[lo:lo + n])
        vs.append(v[lo:lo + n])
        sl.append(slots_for(tab.block_tables[b], lo, n))
    return (torch.cat(ks).contiguous(), torch.cat(vs).contiguous(),
            np.concatenate(sl).astype(np.int32))


def decode_lens(s: Spec) -> np.ndarray:
    """Context lengths seen by the decode step (prefill + appended tokens)."""
    return (seq_lens(s) + s.append_tokens).astype(np.int32)


def softmax_scale(s: Spec) -> float:
    return float(np.float32(1.0 / math.sqrt(s.head_dim)))
