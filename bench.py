#!/usr/bin/env python
"""Benchmark of the paged, quantized KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--kv-dtype bf16|fp16|fp8_e4m3|fp8_e5m2|fp4] [--second-kv FMT|none]
                    [--split-blocks N] [--impl ours|reference]

One step = one decode step of one attention layer over the whole batch:
kv_cache_write of one new token per sequence, then paged_decode_attention of
every sequence over its cache (the write, the split-K decode and its
log-sum-exp merge). Inputs are seeded synthetic data of the workload's shapes,
resident in HBM when timing starts. Prints one JSON line (rank 0).

The default workload is the Llama-3.1-70B-shaped single-GPU layer (16
sequences of 24k-40k tokens, 64 q / 8 KV heads, head_dim 128, four sequences
sharing a 4096-token prefix) with split-K over 512-token chunks, bf16 KV; the
same workload with an FP8 E4M3 cache (same inputs) is measured in the same run
and reported as the nested "fp8_e4m3" object of the same line. Every line
carries the output error of the GPU decode against the CPU oracle on a sample
of sequences ("oracle_error").

N > 1 (torchrun, one process per GPU): every rank runs its own replica of the
workload (weak scaling, no collective on the data path); the timed region is
bracketed by barriers and the time taken is the maximum over ranks.

--impl reference times the CPU oracle (the fp64 restatement used by the tests)
on a bounded sample of the same workload on the host cores.

--op copy_blocks | swap measures the whole-block moves instead (copy-on-write
copies inside the cache; swap of blocks to pinned host memory and back) on the
workload's cache format; one JSON line of the same shape.

--op prefill measures chunked-prefill attention: 16 sequences (Llama-3-8B
shaped, 32 q / 8 KV heads, head_dim 128), each with a prefix of U[0, 7680]
cached tokens and a 512-token chunk; a step writes the chunk's K/V into the
cache and runs the causal attention of its queries over the whole context.

--op write measures the cache write alone: the FP4 + outlier chunked write of
the fp4 workload (512 tokens of each of 256 sequences per call) against its
bytes, with the FP8 single-token append of the fp8 workload nested.

--op read_probe measures the decode's paged gather without its math (the read
ceiling): the workload's tables and an identity table (contiguous reads).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "paged decode-attn KV GB/s (frac of B200 HBM peak); decode tok/s per layer"
UNIT = "GB/s"
KV_NAMES = {"fp16": W.DT_FP16, "bf16": W.DT_BF16, "fp8_e4m3": W.DT_FP8_E4M3, "fp8_e5m2": W.DT_FP8_E5M2,
            "fp4": W.DT_FP4}
DT_LABEL = {W.DT_FP16: "fp16", W.DT_BF16: "bf16", W.DT_FP8_E4M3: "fp8_e4m3", W.DT_FP8_E5M2: "fp8_e5m2",
            W.DT_FP4: "fp4_e2m1"}
DESCR = {
    "tiny": "tiny decode step: 4 seqs, ctx {17,33,64,100}, 8 q / 2 kv heads, head_dim 64, fp16 KV",
    "llama8b": "Llama-3-8B-shaped decode layer: 64 seqs, ctx U[512,4096], 32 q / 8 kv heads, head_dim 128, "
               "block 16, random blocks of a 40k-block pool",
    "fp8": "Llama-3-8B-shaped decode layer, FP8 KV with per-block-per-head absmax scales: 128 seqs, "
           "ctx U[1024,8192]",
    "llama70b": "Llama-3.1-70B-shaped layer: 16 seqs, ctx U[24576,40960], 64 q / 8 kv heads, head_dim 128, "
                "seqs 0-3 share a 4096-token prefix",
    "fp4": "FP4 E2M1 KV with 3.2-sigma fp16 outlier channels: 256 seqs, ctx log-uniform [1024,65536], "
           "32 q / 8 kv heads, head_dim 128, prefill written in 512-token chunks",
}
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# workload on the device
# ---------------------------------------------------------------------------

def bench_spec(name: str, kv_name: str | None, batch: int | None = None, pool: int | None = None,
               q_len: int = 1) -> W.Spec:
    """The workload as bench.py runs it; batch / pool cut it down for profiling."""
    s = W.spec(name, kv_dtype=KV_NAMES[kv_name] if kv_name else None, batch=batch)
    if pool:
        s.pool_blocks = pool
    s.append_tokens = q_len  # every step appends q_len tokens per sequence
    if s.kv_dtype in (W.DT_FP16, W.DT_BF16):
        s.q_dtype = s.kv_dtype  # 16-bit caches take queries of their own type
    return s


def decode_passes(q_len: int, G: int) -> int:
    """Decode passes of a multi-query step: up to 16 query rows (G heads x tokens) per KV read."""
    kp = min(q_len, max(1, 16 // G))
    return -(-q_len // kp)


def per_token_bytes(s: W.Spec) -> int:
    """Algorithmic KV bytes of one token (all KV heads, K and V, with its share of
    the scales / outlier buffers of the cache layout)."""
    H, D = s.num_kv_heads, s.head_dim
    if s.kv_dtype in (W.DT_FP16, W.DT_BF16):
        return H * 2 * D * 2
    if s.kv_dtype in (W.DT_FP8_E4M3, W.DT_FP8_E5M2):
        return H * 2 * D + H * 16 // 16
    return H * 2 * (D // 2 + D // 16 + 4 * 2) + H * 16 // 16


def unique_tokens(s: W.Spec) -> int:
    """Context tokens of a decode step, a shared prefix counted once."""
    tot = int(W.decode_lens(s).sum())
    if s.shared_prefix_seqs:
        tot -= s.shared_prefix_tokens * (min(s.shared_prefix_seqs, s.batch) - 1)
    return tot


def step_bytes(s: W.Spec, q_len: int) -> dict:
    """Algorithmic bytes of one decode call: unique KV bytes, q + out, block-table entries."""
    kv = unique_tokens(s) * per_token_bytes(s)
    qo = 2 * s.batch * q_len * s.num_q_heads * s.head_dim * 2
    tables = int(sum(W.nblocks(int(L)) for L in W.decode_lens(s))) * 4 + s.batch * 4
    return {"kv": kv, "q_out": qo, "tables": tables, "decode_total": kv + qo + tables}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def generate_kv(s: W.Spec, seqs, threads: int = 0, ahead: int = 8):
    """Yield seq_kv(s, b) for b in seqs, in order, computed by a few threads ahead."""
    import concurrent.futures as cf
    seqs = list(seqs)
    threads = threads or max(1, min(16, (os.cpu_count() or 2) - 1))
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        futs = {}
        for i, b in enumerate(seqs):
            for jj in range(i, min(len(seqs), i + ahead)):
                if jj not in futs:
                    futs[jj] = ex.submit(W.seq_kv, s, seqs[jj])
            yield futs.pop(i).result()


class Setup:
    """Cache prefilled with the workload, plus one decode step's inputs, on `device`."""

    def __init__(self, s: W.Spec, device, split_blocks: int, q_len: int = 1, prefill: bool = False,
                 kv_list=None, keep_kv: bool = False):
        """kv_list: the per-sequence host (k, v) of an earlier Setup of the same
        workload (same input dtype), reused instead of drawn again; keep_kv keeps
        this Setup's in self.kv_list."""
        import paged_quantized_kv_cache_b200 as pq
        self.pq = pq
        self.s = s
        self.device = device
        tab = W.tables(s)
        self.tab = tab
        self.lens0 = W.seq_lens(s)
        self.lens = W.decode_lens(s)
        self.q_len = q_len
        self.prefill = prefill  # the step's q_len tokens attend by the chunked-prefill kernel
        self.cache = pq.allocate_cache(s.kv_dtype, tab.num_blocks, s.num_kv_heads, s.head_dim, device=device,
                                       fill=0xFF)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        in_dt = W.TORCH_DTYPE[W.input_dtype(s)]
        # prefill: generate per sequence on the host (seeded, a few threads
        # ahead), write with the GPU in the workload's write-call sizes
        newk, newv = [], []
        self.kv_list = [] if keep_kv else None
        source = kv_list if kv_list is not None else generate_kv(s, range(s.batch))
        for b, (k, v) in enumerate(source):
            k = k.to(in_dt)
            v = v.to(in_dt)
            if keep_kv:
                self.kv_list.append((k, v))
            L0 = int(self.lens0[b])
            lo = s.shared_prefix_tokens if (0 < b < s.shared_prefix_seqs) else 0
            kd, vd = k.to(device), v.to(device)
            step = s.chunk_tokens or L0
            for c0 in range(lo, L0, step):
                c1 = min(L0, c0 + step)
                sl = torch.from_numpy(W.slots_for(tab.block_tables[b], c0, c1 - c0)).to(device)
                pq.kv_cache_write(kd[c0:c1].contiguous(), vd[c0:c1].contiguous(), sl, self.cache, self.err)
            newk.append(k[L0:L0 + q_len])
            newv.append(v[L0:L0 + q_len])
        torch.cuda.synchronize(device)
        if int(self.err.item()) != 0:
            raise RuntimeError("prefill raised device error bits %d" % int(self.err.item()))
        self.k_new = torch.cat(newk).contiguous()
        self.v_new = torch.cat(newv).contiguous()
        self.slots_new = np.concatenate([W.slots_for(tab.block_tables[b], int(self.lens0[b]), q_len)
                                         for b in range(s.batch)]).astype(np.int32)
        self.q = W.query(s) if q_len == 1 else W.multi_query(s, q_len)
        self.split_blocks = split_blocks
        self.scale = W.softmax_scale(s)
        # The step's inputs (q, new k / v, slots, block tables, lengths) live in
        # one packed buffer so the end-to-end leg moves them with one copy.
        parts = [("q", self.q), ("k", self.k_new), ("v", self.v_new),
                 ("slots", torch.from_numpy(self.slots_new)), ("bt", torch.from_numpy(tab.block_tables)),
                 ("lens", torch.from_numpy(self.lens))]
        offs, total = {}, 0
        for name, t in parts:
            offs[name] = total
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        self.h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
        for name, t in parts:
            n = t.numel() * t.element_size()
            self.h_in[offs[name]:offs[name] + n].copy_(t.contiguous().view(-1).view(torch.uint8))
        # two device copies of the inputs and outputs, so that the end-to-end
        # leg can copy one step's inputs in while the previous step computes
        self.d_in_sets, self._views = [], []
        for _ in range(2):
            d_in = torch.empty(total, dtype=torch.uint8, device=device)
            d_in.copy_(self.h_in)
            views = {}
            for name, t in parts:
                n = t.numel() * t.element_size()
                views[name] = d_in[offs[name]:offs[name] + n].view(t.dtype).view(t.shape)
            self.d_in_sets.append(d_in)
            self._views.append(views)
        self.h2d_bytes = sum(t.numel() * t.element_size() for _, t in parts)
        self.d_outs = [torch.empty_like(self._views[0]["q"]) for _ in range(2)]
        self.use(0)
        if prefill:
            self.ws = None
            self.cu = torch.arange(0, (s.batch + 1) * q_len, q_len, dtype=torch.int32, device=device)
        else:
            self.ws = pq.multi_query_decode_workspace(s.batch, q_len, s.num_q_heads, s.num_kv_heads, s.head_dim,
                                                      tab.max_blocks, split_blocks, device=device)

    def use(self, i: int):
        """Make input / output set i the one write() and decode() use."""
        v = self._views[i]
        self.d_in = self.d_in_sets[i]
        self.d_q, self.d_k, self.d_v = v["q"], v["k"], v["v"]
        self.d_slots, self.d_bt, self.d_lens = v["slots"], v["bt"], v["lens"]
        self.d_out = self.d_outs[i]

    def write(self):
        self.pq.kv_cache_write(self.d_k, self.d_v, self.d_slots, self.cache, self.err)

    def decode(self):
        if self.prefill:
            s = self.s
            self.pq.paged_prefill_attention(self.d_q.view(-1, s.num_q_heads, s.head_dim), self.cu, self.q_len,
                                            self.cache, self.d_bt, self.d_lens, self.scale,
                                            self.d_out.view(-1, s.num_q_heads, s.head_dim), self.err)
        elif self.q_len == 1:
            self.pq.paged_decode_attention(self.d_q, self.cache, self.d_bt, self.d_lens, self.scale, self.d_out,
                                           self.ws, self.err, split_blocks=self.split_blocks)
        else:
            self.pq.paged_multi_query_decode_attention(self.d_q, self.cache, self.d_bt, self.d_lens, self.scale,
                                                       self.d_out, self.ws, self.err,
                                                       split_blocks=self.split_blocks)

    def prefill_flops(self) -> float:
        """Causal attention flops of the step's query chunk: 4 * Hq * D per
        (query token, visible position)."""
        s, C = self.s, self.q_len
        pre = self.lens.astype(np.int64) - C
        return 4.0 * s.num_q_heads * s.head_dim * float(np.sum(C * pre + C * (C + 1) // 2))

    def unique_tokens(self) -> int:
        return unique_tokens(self.s)

    def step_bytes(self) -> dict:
        return step_bytes(self.s, self.q_len)


# ---------------------------------------------------------------------------
# clocks (NVML, sampled during the timed region)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.ok = False
        self.samples = []
        self.reasons = 0
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._t = None

    def _sample_once(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        try:
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.reasons |= int(r) & ~0x1

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample_once()
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()
        if self.ok and len(self.samples) < 3:
            for _ in range(3):
                try:
                    self._sample_once()
                except Exception:
                    pass

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("decode.cu", "decode.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "paged_quantized_kv_cache_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kv_name: str, split_blocks: int, q_len: int = 1) -> int | None:
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken from the current kernel source with the same split (one query token
    per sequence: the summaries are of the single-token decode)."""
    p = os.path.join(ROOT, "profiles", "decode_traffic_%s_%s.txt" % (workload, kv_name))
    if q_len != 1 or not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if "=" in line and not line.startswith("#"):
            k, v = line.strip().split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_hash") != decode_source_hash():
        return None
    if int(vals.get("split_blocks", "0")) != split_blocks:
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over the ranks of the default process group."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

class OracleSample:
    """The oracle's decode (gather through the tables, dequantize, fp64
    attention) over a bounded sample of the workload's sequences. The sample's
    cache is written by the oracle itself through the same write calls as the
    GPU cache of bench.py: the prefill in the workload's call sizes, then the
    step's appended token as its own call (for FP8 that call may grow the
    block's scale and re-encode its codes)."""

    def __init__(self, s: W.Spec, nseq: int):
        import oracle
        self.oracle = oracle
        self.s = s
        lens = W.decode_lens(s)
        lens0 = W.seq_lens(s)
        tab = W.tables(s)
        order = [int(i) for i in np.argsort(lens, kind="stable")]
        # a spread of lengths: shortest, longest, then alternating inwards
        pick, lo, hi = [], 0, len(order) - 1
        while lo <= hi:
            pick.append(order[lo]); lo += 1
            if lo <= hi:
                pick.append(order[hi]); hi -= 1
        sample = sorted(pick[:max(1, min(nseq, len(pick)))])
        need = sum(W.nblocks(int(lens[b])) for b in sample)
        self.c = oracle.Cache(s.kv_dtype, need, s.num_kv_heads, s.head_dim)
        self.bt = np.full((len(sample), tab.max_blocks), -1, np.int32)
        nxt = 0
        in_dt = W.TORCH_DTYPE[W.input_dtype(s)]
        for i, b in enumerate(sample):
            nb = W.nblocks(int(lens[b]))
            self.bt[i, :nb] = np.arange(nxt, nxt + nb, dtype=np.int32)
            nxt += nb
            k, v = W.seq_kv(s, b)
            k, v = k.to(in_dt), v.to(in_dt)
            L0, L = int(lens0[b]), int(lens[b])
            step = s.chunk_tokens or L0
            for c0, c1 in [(c, min(L0, c + step)) for c in range(0, L0, step)] + ([(L0, L)] if L > L0 else []):
                oracle.kv_cache_write(self.c, k[c0:c1].contiguous(), v[c0:c1].contiguous(),
                                      W.slots_for(self.bt[i], c0, c1 - c0))
        self.q = W.query(s)[sample].contiguous()
        self.lens = lens[sample].astype(np.int32)
        self.sample = sample
        self.tokens = int(self.lens.sum())

    def step(self):
        return self.oracle.paged_decode(self.c, self.q, self.bt, self.lens, W.softmax_scale(self.s))[0]

    def describe(self, reps: int, per: float) -> str:
        return ("%d of %d sequences (%d tokens, lengths %d..%d); oracle decode (gather, dequantize, fp64 "
                "attention) timed %d times, %.3f s each" % (len(self.sample), self.s.batch, self.tokens,
                                                            int(self.lens.min()), int(self.lens.max()), reps, per))

    def errors(self, gpu_out: torch.Tensor) -> dict:
        """Output error of the GPU decode on the sample sequences against the
        oracle (fp64, unrounded), with the tolerance the parity tests use."""
        ref = self.step()
        got = gpu_out[self.sample].double().cpu().numpy()
        fp4 = self.s.kv_dtype == W.DT_FP4
        atol, rtol = (5e-3 if fp4 else 2e-3), 1e-2
        d = np.abs(got - ref)
        big = np.abs(ref) >= 0.1 * np.abs(ref).max()
        return {"max_abs_err": float(d.max()),
                "max_rel_err": float((d[big] / np.abs(ref[big])).max()),
                "tol_used": float((d / (atol + rtol * np.abs(ref))).max()),
                "atol": atol, "rtol": rtol,
                "sample": "%d of %d sequences, all %d x %d outputs each; max_rel_err over outputs with |ref| >= "
                          "0.1 max|ref|; tol_used = max |gpu - ref| / (atol + rtol |ref|) (pass <= 1)"
                          % (len(self.sample), self.s.batch, self.s.num_q_heads, self.s.head_dim)}


def oracle_baseline(s: W.Spec, budget_s: float, nseq: int, o: "OracleSample | None" = None) -> dict:
    """cpu_baseline: the oracle as it stands, timed for about budget_s seconds."""
    o = o or OracleSample(s, nseq)
    t_total, reps = 0.0, 0
    while reps < 1 or (t_total < budget_s and reps < 100000):
        t0 = time.perf_counter()
        o.step()
        t_total += time.perf_counter() - t0
        reps += 1
    per = t_total / reps
    return {"value": o.tokens * per_token_bytes(s) / per / 1e9, "unit": UNIT, "cores": o.oracle.num_threads(),
            "cpu_model": cpu_model(), "kind": "oracle", "sample": o.describe(reps, per)}


def run_reference(args) -> None:
    """The oracle on the host cores, same metric and workload; each step is the
    oracle decode over a sample small enough for W + K steps to take minutes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    s = bench_spec(args.workload, args.kv_dtype, args.batch, args.pool_blocks)
    nseq = args.ref_seqs
    budget = 150.0
    while True:
        o = OracleSample(s, nseq)
        t0 = time.perf_counter()
        o.step()
        one = time.perf_counter() - t0
        if (args.steps + args.warmup) * one <= budget or nseq == 1:
            break
        nseq = max(1, nseq // 2)
    for _ in range(args.warmup):
        o.step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        o.step()
        times.append(time.perf_counter() - t0)
    per = statistics.mean(times)
    value = o.tokens * per_token_bytes(s) / per / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args, s),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.oracle.num_threads(), "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": o.describe(args.steps, per)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(args, s: W.Spec) -> dict:
    """The workload's description; the same keys for our arm and the reference arm."""
    b = step_bytes(s, args.q_len)
    d = {"workload": args.workload + ": " + DESCR[args.workload] + "; KV " + DT_LABEL[s.kv_dtype] +
         ("; step = append 1 token per sequence + paged decode" if args.q_len == 1 else
          "; step = append %d tokens per sequence + multi-query decode verifying them (speculative decoding)"
          % args.q_len), "batch": s.batch, "q_len": args.q_len,
         "num_q_heads": s.num_q_heads, "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim,
         "block_size": 16, "kv_dtype": DT_LABEL[s.kv_dtype], "split_blocks": args.split_blocks,
         "parallelism": "replicas (one independent batch per GPU)",
         "context_tokens": int(W.decode_lens(s).sum()), "kv_bytes_per_step": b["kv"]}
    d["l2"] = ("inputs larger than L2: %.0f MB of KV read per step vs 126 MB L2; no flush"
               % (b["kv"] / 1e6)) if b["kv"] > 2 * L2_BYTES else \
        "KV smaller than L2 (%.1f MB): numbers include L2 hits" % (b["kv"] / 1e6)
    return d


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def measure_decode(args, s: W.Spec, device, world: int, kv_list=None, keep_kv: bool = False):
    """Time K decode steps of workload s (write + decode, back to back), then
    the calls' own durations, then the end-to-end leg. Returns (dict, Setup)."""
    st = Setup(s, device, args.split_blocks, args.q_len, kv_list=kv_list, keep_kv=keep_kv)
    stream = torch.cuda.current_stream(device)
    for _ in range(max(args.warmup, 3)):
        st.write()
        st.decode()
    torch.cuda.synchronize(device)
    K = args.steps
    clocks = ClockSampler(device.index)
    # the timed region: K steps back to back (nothing between the kernels, so
    # each launch overlaps the previous kernel's tail as programmed)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(device)
    clocks.start()
    e0.record(stream)
    for i in range(K):
        st.write()
        st.decode()
    e1.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    barrier(world)
    if int(st.err.item()) != 0:
        raise RuntimeError("device error bits %d during the timed steps" % int(st.err.item()))
    total_ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_step = total_ms / K
    # then K more steps with events around each call, for the kernels' own times
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        ev[i][0].record(stream)
        st.write()
        ev[i][1].record(stream)
        st.decode()
        ev[i][2].record(stream)
    torch.cuda.synchronize(device)
    dec_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(K))
    wr_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))
    b = st.step_bytes()
    peaks = measured_peaks()
    achieved = b["decode_total"] / (dec_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": profiled_traffic(args.workload, DT_LABEL[s.kv_dtype], args.split_blocks, args.q_len),
                "kernel": "paged_decode_kernel", "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, "
                "a read+write copy)", "bytes_per_launch": b["decode_total"], "avg_launch_ms": dec_ms,
                "timing": "CUDA events around each decode call (one decode kernel per pass, which also merges the "
                          "split pairs) over K further steps"}
    e2e = run_e2e(st, args, world) if not args.no_e2e else None
    value = b["kv"] * world / (ms_step * 1e-3) / 1e9
    m = {"value": value, "ms_per_step": ms_step,
         "frac_of_hbm_peak": value / world / peaks["hbm_gbs"],
         "frac_of_8tbs_spec": value / world / 8000.0,
         "decode_tok_s_per_layer": s.batch * args.q_len * world / (ms_step * 1e-3),
         # the decode call alone (no cache write): B x q_len / t(decode)
         "decode_only_tok_s_per_layer": s.batch * args.q_len * world / (dec_ms * 1e-3),
         "decode_kernel_ms": dec_ms, "write_kernel_ms": wr_ms, "roofline": roofline, "e2e": e2e,
         # per step: cache write, then one decode kernel per pass (it merges the split pairs itself)
         "gpu_launches": (1 + decode_passes(args.q_len, s.num_q_heads // s.num_kv_heads)) * K,
         "clocks": clocks.summary()}
    return m, st


def fp4_outlier_stats(st: Setup) -> dict:
    """Outlier channels the GPU write chose on the fp4 workload, against the
    two planted x16 channels per (KV head, K|V): over every block whose first
    write held all 16 tokens."""
    s = st.s
    idx = st.cache.outliers_idx.view(st.tab.num_blocks, s.num_kv_heads, 2, 8).cpu().numpy()
    planted = W.outlier_channels(s)  # [H][2][2]
    lens0 = W.seq_lens(s)
    ids = np.concatenate([st.tab.block_tables[b, :int(lens0[b]) // 16] for b in range(s.batch)])
    sel = idx[ids][..., :4].astype(np.int64)  # [n][H][2][4], ascending, 0xFF = empty
    c0, c1 = planted[None, :, :, 0, None], planted[None, :, :, 1, None]
    used = sel != 0xFF
    extra = used & (sel != c0) & (sel != c1)
    has0 = (sel == c0).any(-1)
    has1 = (sel == c1).any(-1)
    exact = has0 & has1 & (used.sum(-1) == 2)
    n = int(exact.size)
    return {"blocks_checked": n, "exact": int(exact.sum()), "missed_planted": int((~(has0 & has1)).sum()),
            "with_false_positives": int(extra.any(-1).sum()), "false_positive_channels": int(extra.sum()),
            "what": "(block, KV head, K|V) triples of full blocks; planted = the workload's two x16 channels"}


def run_ours(args) -> None:
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    s = bench_spec(args.workload, args.kv_dtype, args.batch, args.pool_blocks, args.q_len)
    second = args.second_kv
    m, st = measure_decode(args, s, device, world, keep_kv=second is not None)
    line = None
    if rank == 0:
        cpu, errs, oracle_sample = None, None, None
        if args.q_len == 1 and not args.no_oracle_check:
            oracle_sample = OracleSample(s, args.ref_seqs)
            errs = oracle_sample.errors(st.d_out)
        if world == 1 and not args.no_cpu_baseline and args.q_len == 1:
            cpu = oracle_baseline(s, args.cpu_budget, args.ref_seqs, oracle_sample)
        line = {
            "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if s.kv_dtype == W.DT_BF16 else ("fp16" if s.kv_dtype == W.DT_FP16 else
                                                             DT_LABEL[s.kv_dtype] + "->f16"),
            "data": "synthetic", "config": config_dict(args, s)}
        line.update({k: v for k, v in m.items() if k not in ("value", "ms_per_step")})
        line["cpu_baseline"] = cpu
        line["oracle_error"] = errs
        if s.kv_dtype == W.DT_FP4:
            line["outliers"] = fp4_outlier_stats(st)
    kv_list = st.kv_list
    del st
    torch.cuda.empty_cache()
    if second is not None:
        # the same workload and inputs with the second cache format, in the same run
        s2 = bench_spec(args.workload, second, args.batch, args.pool_blocks, args.q_len)
        m2, st2 = measure_decode(args, s2, device, world, kv_list=kv_list)
        del kv_list
        if rank == 0:
            sub = {"kv_dtype": DT_LABEL[s2.kv_dtype], "dtype": DT_LABEL[s2.kv_dtype] + "->f16",
                   "config": config_dict(args, s2)}
            sub.update(m2)
            if args.q_len == 1 and not args.no_oracle_check:
                sub["oracle_error"] = OracleSample(s2, args.ref_seqs).errors(st2.d_out)
            line[DT_LABEL[s2.kv_dtype]] = sub
        del st2
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(st: Setup, args, world: int, per_step=None, unit: str = UNIT, scale: float = 1e9) -> dict:
    """Same step through the public API from pinned host buffers, as a serving
    loop runs it: every step copies its inputs in (q, the new tokens' k / v,
    slots, block tables, lengths; one packed copy) and its output back. The
    copies run on their own streams, so step i + 1's inputs travel in and step
    i's output travels out while step i computes (two device buffer sets);
    the timed region spans the first input copy to the last output copy."""
    dev = st.device
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h_outs = [torch.empty(st.d_outs[0].shape, dtype=st.d_outs[0].dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = st.h2d_bytes
    d2h = h_outs[0].numel() * h_outs[0].element_size()

    def step(i):
        b = i & 1
        if i >= 2:
            s_in.wait_event(ev_comp[b])  # step i - 2 has read this input set
        with torch.cuda.stream(s_in):
            st.d_in_sets[b].copy_(st.h_in, non_blocking=True)
        ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])  # step i - 2's output has left this buffer
        st.use(b)
        st.write()
        st.decode()
        ev_comp[b].record(comp)
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            h_outs[b].copy_(st.d_outs[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    K = max(1, args.steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(s_in)
    for i in range(K):
        step(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(world)
    st.use(0)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / K
    work = st.step_bytes()["kv"] if per_step is None else per_step
    return {"value": work * world / (ms * 1e-3) / scale, "unit": unit, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "inputs of step i+1 copied in and output of step i copied out while step i computes"}

def run_block_op(args) -> None:
    """copy_blocks: n random (src, dst) pairs of the workload's pool per step.
    swap: n blocks out to pinned host records, then back in, per step; the host
    link's reference is a plain cudaMemcpyAsync of the same bytes each way."""
    import oracle
    import paged_quantized_kv_cache_b200 as pq
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    s = bench_spec(args.workload, args.kv_dtype, None, args.pool_blocks)
    nb = s.pool_blocks
    g = pq.allocate_cache(s.kv_dtype, nb, s.num_kv_heads, s.head_dim, device=dev)
    for a in g.arrays():
        if a is not None:
            a.copy_(torch.randint(0, 256, a.shape, dtype=torch.uint8, device=dev))
    rec = pq.block_record_bytes(s.kv_dtype, s.num_kv_heads, s.head_dim)
    rng = np.random.default_rng(100 + rank)
    n = args.op_blocks
    ids = rng.choice(nb, size=2 * n, replace=False).astype(np.int32)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    if args.op == "copy_blocks":
        pairs_h = torch.from_numpy(ids.reshape(2, n).T.copy()).pin_memory()
        pairs = pairs_h.to(dev)
        step = lambda: pq.copy_blocks(g, pairs, err)  # noqa: E731
        bytes_step = 2 * n * rec
        metric = "copy_blocks GB/s (bytes read + written; copy-on-write block copies)"
    else:
        host = torch.empty(n * rec, dtype=torch.uint8).pin_memory()
        blk = torch.from_numpy(ids[:n].copy()).to(dev)
        blk_in = torch.from_numpy(ids[n:].copy()).to(dev)

        def step():
            pq.swap_out(g, blk, host, err)
            pq.swap_in(g, blk_in, host, err)
        bytes_step = 2 * n * rec
        metric = "swap GB/s over the host link (blocks out to pinned host records and back in)"
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(world)
    if int(err.item()) != 0:
        raise RuntimeError("device error bits %d" % int(err.item()))
    ms = max_over_ranks(e0.elapsed_time(e1), world) / K
    value = bytes_step * world / (ms * 1e-3) / 1e9
    peaks = measured_peaks()
    if args.op == "copy_blocks":
        roofline = {"bound": "hbm", "achieved": value / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": value / world / peaks["hbm_gbs"], "traffic": None, "kernel": "block_move_kernel<copy>",
                    "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, a read+write copy)"}
        # e2e: the pairs come from pinned host memory every step, the error flag goes back
        h_err = torch.empty(1, dtype=torch.int32).pin_memory()

        def e2e_step():
            pairs.copy_(pairs_h, non_blocking=True)
            step()
            h_err.copy_(err, non_blocking=True)
        h2d, d2h = pairs_h.numel() * 4, 4
    else:
        # reference for the host link: cudaMemcpyAsync of the same bytes each way
        dbuf = torch.empty(n * rec, dtype=torch.uint8, device=dev)
        for _ in range(3):
            host.copy_(dbuf, non_blocking=True)
            dbuf.copy_(host, non_blocking=True)
        torch.cuda.synchronize(dev)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for _ in range(K):
            host.copy_(dbuf, non_blocking=True)
            dbuf.copy_(host, non_blocking=True)
        m1.record(stream)
        torch.cuda.synchronize(dev)
        memcpy_gbs = bytes_step / (m0.elapsed_time(m1) / K * 1e-3) / 1e9
        roofline = {"bound": "host link", "achieved": value / world, "peak": memcpy_gbs, "unit": "GB/s",
                    "frac": value / world / memcpy_gbs, "traffic": None, "kernel": "block_move_kernel<to/from host>",
                    "peak_source": "cudaMemcpyAsync of the same bytes D2H + H2D (pinned), measured in this run"}
        e2e_step, h2d, d2h = step, n * rec, n * rec
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(K):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world) / K
    e2e = {"value": bytes_step * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_e2e,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            # the oracle's block copy (numpy slices) on a bounded host-memory sample
            nsm = min(n, 256)
            oc = oracle.Cache(s.kv_dtype, 2 * nsm, s.num_kv_heads, s.head_dim, poison=False)
            pr = np.stack([np.arange(nsm), np.arange(nsm) + nsm], axis=1)
            reps, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < min(args.cpu_budget, 5.0):
                oracle.copy_blocks(oc, pr)
                reps += 1
            dt = time.perf_counter() - t0
            cpu = {"value": 2 * nsm * rec * reps / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                   "sample": "%d block copies of %d bytes, repeated for %.1f s" % (nsm, rec, dt)}
        line = {
            "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": "%s cache (%s, %d KV heads, head_dim %d, pool %d blocks): %d blocks of %d "
                                   "bytes per step" % (args.workload, DT_LABEL[s.kv_dtype], s.num_kv_heads,
                                                       s.head_dim, nb, n, rec),
                       "op": args.op, "blocks_per_step": n, "record_bytes": rec,
                       "l2": "%.0f MB moved per step vs 126 MB L2" % (bytes_step / 1e6)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": (1 if args.op == "copy_blocks" else 2) * K, "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def _init_dist(local: int):
    torch.cuda.set_device(local)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return torch.device("cuda", local)


def _end_dist(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def _time_calls(fn, K: int, warmup: int, device, world: int):
    """K calls back to back between two events (after warm-up); ms per call (max over ranks) and clocks."""
    stream = torch.cuda.current_stream(device)
    for _ in range(max(warmup, 3)):
        fn()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device.index)
    barrier(world)
    torch.cuda.synchronize(device)
    clocks.start()
    e0.record(stream)
    for _ in range(K):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world) / K, clocks.summary()


def _kv_rows(s: W.Spec, rows, threads: int = 16):
    """(k, v) host tensors of write rows [(b, start, n)], drawn by W.write_kv in threads, concatenated."""
    import concurrent.futures as cf
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(lambda r: W.write_kv(s, *r), rows))
    return torch.cat([p[0] for p in parts]).contiguous(), torch.cat([p[1] for p in parts]).contiguous()


def write_call_bytes(kv_dtype: int, T: int, H: int, D: int, blocks: int, reencode_tokens: int = 0) -> int:
    """Algorithmic bytes of one write call of T tokens touching `blocks` (block, call)
    pairs: K/V read (bf16) + slots read + codes / scales / outlier buffers written,
    plus the read and rewrite of `reencode_tokens` earlier FP8 codes."""
    b = T * H * 2 * D * 2 + T * 4
    if kv_dtype in (W.DT_FP16, W.DT_BF16):
        return b + T * H * 2 * D * 2
    if kv_dtype in (W.DT_FP8_E4M3, W.DT_FP8_E5M2):
        return b + T * H * 2 * D + blocks * H * 16 + 2 * reencode_tokens * H * 2 * D
    return b + T * H * 2 * (D // 2 + D // 16 + 4 * 2) + blocks * H * 2 * 8


def run_write(args) -> None:
    """The cache write on its own. Main line: the FP4 + outlier chunked write of
    the fp4 workload (one call = the first 512-token chunk of all 256 sequences,
    131,072 tokens into random blocks of the 1M-block pool), against its bytes.
    Nested: the FP8 E4M3 single-token append of the fp8 workload (128 tokens,
    one per sequence, into partly filled blocks), a latency-bound call."""
    import oracle
    import paged_quantized_kv_cache_b200 as pq
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    dev = _init_dist(local)
    C = 512
    s = bench_spec("fp4", None, args.batch, args.pool_blocks)
    B, H, D = s.batch, s.num_kv_heads, s.head_dim
    tab = W.tables(s)
    rows = [(b, 0, C) for b in range(B)]
    k_h, v_h = _kv_rows(s, rows)
    slots_h = np.concatenate([W.slots_for(tab.block_tables[b], 0, C) for b in range(B)]).astype(np.int32)
    cache = pq.allocate_cache(s.kv_dtype, tab.num_blocks, H, D, device=dev, fill=0xFF)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    k_d, v_d, sl_d = k_h.to(dev), v_h.to(dev), torch.from_numpy(slots_h).to(dev)
    call = lambda: pq.kv_cache_write(k_d, v_d, sl_d, cache, err)  # noqa: E731
    ms, clocks = _time_calls(call, args.steps, args.warmup, dev, world)
    if int(err.item()) != 0:
        raise RuntimeError("device error bits %d" % int(err.item()))
    T = B * C
    nbytes = write_call_bytes(s.kv_dtype, T, H, D, T // 16)
    peaks = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": "write_fp4_kernel",
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, a read+write copy)",
                "bytes_per_launch": nbytes, "avg_launch_ms": ms,
                "timing": "K calls back to back between two CUDA events (one kernel per call)"}
    # parity of the timed call on a sample of sequences: every byte of their blocks
    nsm = min(4, B)
    oc = oracle.Cache(s.kv_dtype, nsm * (C // 16), H, D)
    obt = np.arange(nsm * (C // 16), dtype=np.int32).reshape(nsm, C // 16)
    for i in range(nsm):
        oracle.kv_cache_write(oc, k_h[i * C:(i + 1) * C], v_h[i * C:(i + 1) * C], W.slots_for(obt[i], 0, C))
    g_arrays = [a.view(tab.num_blocks, -1).cpu().numpy() if a is not None else None for a in cache.arrays()]
    for i in range(nsm):
        ids = tab.block_tables[i, :C // 16]
        for ga, oa in zip(g_arrays, oc.arrays()):
            if ga is not None and not np.array_equal(ga[ids], oa.reshape(oc.nb, -1)[obt[i]]):
                raise RuntimeError("write parity: GPU cache bytes differ from the oracle's")
    # end to end: the call's inputs from pinned host memory every call, the error flag back
    k_p, v_p, sl_p = k_h.pin_memory(), v_h.pin_memory(), torch.from_numpy(slots_h).pin_memory()
    h_err = torch.empty(1, dtype=torch.int32).pin_memory()

    def e2e_call():
        k_d.copy_(k_p, non_blocking=True)
        v_d.copy_(v_p, non_blocking=True)
        sl_d.copy_(sl_p, non_blocking=True)
        call()
        h_err.copy_(err, non_blocking=True)
    ms_e2e, _ = _time_calls(e2e_call, max(3, min(args.steps, 50)), 3, dev, world)
    e2e = {"value": nbytes * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_e2e,
           "h2d_bytes_per_step": 2 * T * H * D * 2 + T * 4, "d2h_bytes_per_step": 4}

    # nested: FP8 E4M3 single-token append (fp8 workload), steady state
    s8 = bench_spec("fp8", "fp8_e4m3", None, None)
    tab8 = W.tables(s8)
    L0 = W.seq_lens(s8)
    c8 = pq.allocate_cache(s8.kv_dtype, tab8.num_blocks, H, D, device=dev, fill=0xFF)
    pre = [(b, int(L0[b]) // 16 * 16, int(L0[b]) % 16) for b in range(s8.batch) if int(L0[b]) % 16]
    if pre:  # the earlier tokens of each partly filled block
        kp, vp = _kv_rows(s8, pre)
        slp = np.concatenate([W.slots_for(tab8.block_tables[b], st0, n) for b, st0, n in pre]).astype(np.int32)
        pq.kv_cache_write(kp.to(dev), vp.to(dev), torch.from_numpy(slp).to(dev), c8, err)
    ka, va = _kv_rows(s8, [(b, int(L0[b]), 1) for b in range(s8.batch)])
    sla = torch.from_numpy(np.array([W.slots_for(tab8.block_tables[b], int(L0[b]), 1)[0]
                                     for b in range(s8.batch)], np.int32)).to(dev)
    ka, va = ka.to(dev), va.to(dev)
    ms8, _ = _time_calls(lambda: pq.kv_cache_write(ka, va, sla, c8, err), args.steps, args.warmup, dev, world)
    if int(err.item()) != 0:
        raise RuntimeError("device error bits %d" % int(err.item()))
    nb8 = write_call_bytes(s8.kv_dtype, s8.batch, H, D, s8.batch)
    append = {"what": "fp8 workload: 1 token appended to each of 128 sequences (partly filled blocks), E4M3; the "
                      "token is already inside its block's scale after the first call, so the timed calls take "
                      "the path without re-encoding",
              "us_per_call": ms8 * 1e3, "bytes_per_call": nb8, "achieved_gbs": nb8 / (ms8 * 1e-3) / 1e9,
              "bound": "latency (a few KB per SM)"}
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            ocb = oracle.Cache(s.kv_dtype, nsm * (C // 16), H, D)
            reps, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < min(args.cpu_budget, 10.0) or reps == 0:
                for i in range(nsm):
                    oracle.kv_cache_write(ocb, k_h[i * C:(i + 1) * C], v_h[i * C:(i + 1) * C],
                                          W.slots_for(obt[i], 0, C))
                reps += 1
            dt = time.perf_counter() - t0
            cpu = {"value": write_call_bytes(s.kv_dtype, nsm * C, H, D, nsm * C // 16) * reps / dt / 1e9,
                   "unit": "GB/s", "cores": 1, "cpu_model": cpu_model(), "kind": "oracle",
                   "sample": "the oracle's write of %d of the call's %d sequences (%d tokens), %d times in %.1f s"
                             % (nsm, B, nsm * C, reps, dt)}
        line = {
            "metric": "KV cache write GB/s (FP4 E2M1 + fp16 outliers, 512-token chunk write)", "value":
                nbytes * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16->fp4_e2m1", "data": "synthetic",
            "config": {"workload": "fp4 workload's chunked write: the first 512-token chunk of all %d sequences "
                                   "(%d tokens, 8 kv heads, head_dim 128, bf16 in, FP4 E2M1 + E4M3 group scales "
                                   "+ up to 4 fp16 outlier channels out) into random blocks of a %d-block pool"
                                   % (B, T, tab.num_blocks), "tokens": T, "bytes_per_call": nbytes,
                       "l2": "%.0f MB read + written per call vs 126 MB L2; no flush" % (nbytes / 1e6)},
            "roofline": roofline, "parity": "bit-exact against the oracle on %d sequences' blocks" % nsm,
            "cpu_baseline": cpu, "e2e": e2e, "fp8_append": append,
            "gpu_launches": args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    _end_dist(world)


def run_read_probe(args) -> None:
    """The decode's paged gather without its math (pqkv_read_probe), on the
    workload's block tables and on an identity table (contiguous read)."""
    import paged_quantized_kv_cache_b200 as pq
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    dev = _init_dist(local)
    s = bench_spec(args.workload, args.kv_dtype, args.batch, args.pool_blocks)
    tab = W.tables(s)
    lens = W.decode_lens(s)
    cache = pq.allocate_cache(s.kv_dtype, tab.num_blocks, s.num_kv_heads, s.head_dim, device=dev, fill=0x3C)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    chk = torch.zeros(1, dtype=torch.int32, device=dev)
    sl = torch.from_numpy(lens).to(dev)
    nblk = [W.nblocks(int(L)) for L in lens]
    bt_id = np.full_like(tab.block_tables, -1)
    pos = 0
    for b, n in enumerate(nblk):
        bt_id[b, :n] = np.arange(pos, pos + n, dtype=np.int32)
        pos += n
    if pos > tab.num_blocks:
        raise RuntimeError("the identity table needs %d blocks, the pool has %d" % (pos, tab.num_blocks))
    tile = 2 * 16 * {W.DT_FP16: 2 * s.head_dim, W.DT_BF16: 2 * s.head_dim, W.DT_FP4: s.head_dim // 2}.get(
        s.kv_dtype, s.head_dim)
    nbytes = sum(nblk) * s.num_kv_heads * tile
    peaks = measured_peaks()
    res = {}
    for name, bt in (("gather", tab.block_tables), ("contiguous", bt_id)):
        btd = torch.from_numpy(bt).to(dev)
        ms, clocks = _time_calls(lambda: pq.read_probe(cache, btd, sl, chk, err), args.steps, args.warmup, dev,
                                 world)
        res[name] = {"gbs": nbytes / (ms * 1e-3) / 1e9, "ms": ms, "clocks": clocks}
    if int(err.item()) != 0:
        raise RuntimeError("device error bits %d" % int(err.item()))
    if rank == 0:
        g = res["gather"]["gbs"]
        line = {
            "metric": "paged KV gather GB/s (read-only probe: the decode's tile reads without its math)",
            "value": g * world, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": res["gather"]["ms"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u8", "data": "synthetic",
            "config": {"workload": args.workload + ": " + DESCR[args.workload] + "; KV " + DT_LABEL[s.kv_dtype],
                       "tiles_per_call": sum(nblk) * s.num_kv_heads, "tile_bytes": tile, "bytes_per_call": nbytes,
                       "l2": "%.0f MB read per call vs 126 MB L2; no flush" % (nbytes / 1e6)},
            "roofline": {"bound": "hbm", "achieved": g, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": g / peaks["hbm_gbs"], "traffic": None, "kernel": "read_probe_kernel",
                         "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, a read+write copy)"},
            "contiguous_gbs": res["contiguous"]["gbs"], "contiguous_frac": res["contiguous"]["gbs"] / peaks["hbm_gbs"],
            "frac_of_8tbs_spec": g / 8000.0, "cpu_baseline": None,
            "e2e": None, "gpu_launches": 2 * args.steps, "clocks": res["gather"]["clocks"],
            "note": "a measurement of the read ceiling, not a step of the method: no CPU baseline or end-to-end leg",
        }
        print(json.dumps(line), flush=True)
    _end_dist(world)


PREFILL_DESCR = ("chunked prefill, Llama-3-8B-shaped layer: 16 seqs, prefix U[0,7680] cached tokens + a 512-token "
                 "chunk each (written, then causal attention over prefix + chunk), 32 q / 8 kv heads, head_dim 128, "
                 "block 16")


def run_prefill(args) -> None:
    """One step = kv_cache_write of each sequence's 512-token chunk + the
    chunked-prefill attention of its queries over prefix + chunk."""
    import oracle
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    s = bench_spec("prefill", args.kv_dtype, args.batch, args.pool_blocks, q_len=512)
    st = Setup(s, device, 0, q_len=512, prefill=True)
    stream = torch.cuda.current_stream(device)
    for _ in range(max(args.warmup, 3)):
        st.write()
        st.decode()
    torch.cuda.synchronize(device)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(device)
    clocks.start()
    e0.record(stream)
    for i in range(K):
        st.write()
        st.decode()
    e1.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    barrier(world)
    if int(st.err.item()) != 0:
        raise RuntimeError("device error bits %d" % int(st.err.item()))
    ms = max_over_ranks(e0.elapsed_time(e1), world) / K
    # then K more steps with events around each call, for the kernels' own times
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        ev[i][0].record(stream)
        st.write()
        ev[i][1].record(stream)
        st.decode()
        ev[i][2].record(stream)
    torch.cuda.synchronize(device)
    att_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(K))
    wr_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))
    flops = st.prefill_flops()
    value = flops * world / (ms * 1e-3) / 1e12
    peaks = measured_peaks()
    achieved = flops / (att_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": None, "kernel": "paged_prefill_kernel",
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json bf16_tflops, cuBLAS bf16 burst; the f16 "
                "operands of quantized caches run at the same dense rate)",
                "flops_per_launch": flops, "avg_launch_ms": att_ms}
    e2e = None if args.no_e2e else run_e2e(st, argparse.Namespace(steps=min(K, 50)), world, per_step=flops,
                                            unit="TFLOP/s", scale=1e12)
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            # the oracle's prefill of one sequence: a 64-token chunk after 1024 cached tokens
            r2 = np.random.default_rng(3)
            Hq, Hkv, D = s.num_q_heads, s.num_kv_heads, s.head_dim
            L, qn = 1088, 64
            in_dt = W.TORCH_DTYPE[W.input_dtype(s)]
            oc = oracle.Cache(s.kv_dtype, (L + 15) // 16, Hkv, D, poison=False)
            tab = np.arange((L + 15) // 16, dtype=np.int32)[None]
            kk = torch.from_numpy(r2.standard_normal((L, Hkv, D)).astype(np.float32)).to(in_dt)
            vv = torch.from_numpy(r2.standard_normal((L, Hkv, D)).astype(np.float32)).to(in_dt)
            oracle.kv_cache_write(oc, kk, vv, np.arange(L, dtype=np.int32))
            qq = torch.from_numpy(r2.standard_normal((qn, Hq, D)).astype(np.float32)).to(in_dt)
            cuq = np.array([0, qn], np.int32)
            f1 = 4.0 * Hq * D * (qn * (L - qn) + qn * (qn + 1) // 2)
            reps, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < min(args.cpu_budget, 10.0):
                oracle.paged_prefill(oc, qq, cuq, tab, np.array([L], np.int32), st.scale)
                reps += 1
            dt = time.perf_counter() - t0
            cpu = {"value": f1 * reps / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                   "sample": "%d runs of one sequence: a %d-token chunk after %d cached tokens, %s cache, %.1f s"
                             % (reps, qn, L - qn, DT_LABEL[s.kv_dtype], dt)}
        line = {
            "metric": "chunked-prefill attention TFLOP/s (causal, paged cache)", "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if s.kv_dtype == W.DT_BF16 else ("fp16" if s.kv_dtype == W.DT_FP16 else
                                                             DT_LABEL[s.kv_dtype] + "->f16"),
            "data": "synthetic",
            "config": {"workload": PREFILL_DESCR + "; KV " + DT_LABEL[s.kv_dtype], "batch": s.batch, "chunk": 512,
                       "num_q_heads": s.num_q_heads, "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim,
                       "context_tokens": int(st.lens.sum()),
                       "l2": "KV read per step %.0f MB (prefix + chunk) vs 126 MB L2; no flush"
                             % (st.step_bytes()["kv"] / 1e6)},
            "attention_kernel_ms": att_ms, "write_kernel_ms": wr_ms,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 2 * K, "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(DESCR), default="llama70b")
    ap.add_argument("--kv-dtype", choices=sorted(KV_NAMES), default=None)
    ap.add_argument("--second-kv", choices=sorted(KV_NAMES) + ["none"], default=None,
                    help="a second cache format measured on the same workload and inputs, reported as a nested "
                         "object of the same line (default: fp8_e4m3 for the bf16 llama70b workload, else none)")
    ap.add_argument("--split-blocks", type=int, default=None,
                    help="blocks per split-K chunk (default: the workload's; 32 = 512 tokens for llama70b, "
                         "0 = balanced elsewhere)")
    ap.add_argument("--batch", type=int, default=None, help="first N sequences only (profiling subsets)")
    ap.add_argument("--pool-blocks", type=int, default=None, help="smaller block pool (profiling subsets)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-oracle-check", action="store_true", help="skip the output-error statistics")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle timing")
    ap.add_argument("--ref-seqs", type=int, default=None, help="sequences in the oracle sample")
    ap.add_argument("--op", choices=["decode", "copy_blocks", "swap", "prefill", "write", "read_probe"],
                    default="decode")
    ap.add_argument("--op-blocks", type=int, default=4096, help="blocks moved per step (--op copy_blocks|swap)")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per sequence and step (> 1: multi-query decode, speculative verification)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.ref_seqs is None:
        args.ref_seqs = {"tiny": 4, "llama8b": 64, "fp8": 32, "llama70b": 4, "fp4": 16}[args.workload]
    if args.split_blocks is None:
        args.split_blocks = W.spec(args.workload).split_blocks
    if args.second_kv is None:
        base = args.kv_dtype or DT_LABEL[W.spec(args.workload).kv_dtype]
        args.second_kv = "fp8_e4m3" if (args.workload == "llama70b" and base == "bf16"
                                        and args.op == "decode") else None
    elif args.second_kv == "none":
        args.second_kv = None
    if args.impl == "reference":
        run_reference(args)
    elif args.op == "prefill":
        run_prefill(args)
    elif args.op == "write":
        run_write(args)
    elif args.op == "read_probe":
        run_read_probe(args)
    elif args.op != "decode":
        run_block_op(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
