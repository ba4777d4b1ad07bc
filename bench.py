#!/usr/bin/env python
"""Benchmark of the paged, quantized KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--kv-dtype bf16|fp16|fp8_e4m3|fp8_e5m2|fp4] [--impl ours|reference]

One step = one decode step of one attention layer over the whole batch:
kv_cache_write of one new token per sequence, then paged_decode_attention of
every sequence over its cache (the write, the split-K decode and its
log-sum-exp merge). Inputs are seeded synthetic data of the workload's shapes,
resident in HBM when timing starts. Prints one JSON line (rank 0).

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

    def __init__(self, s: W.Spec, device, split_blocks: int, q_len: int = 1, prefill: bool = False):
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
        for b, (k, v) in enumerate(generate_kv(s, range(s.batch))):
            k = k.to(in_dt)
            v = v.to(in_dt)
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
        s = self.s
        tot = int(self.lens.sum())
        if s.shared_prefix_seqs:
            tot -= s.shared_prefix_tokens * (min(s.shared_prefix_seqs, s.batch) - 1)
        return tot

    def step_bytes(self) -> dict:
        s = self.s
        kv = self.unique_tokens() * per_token_bytes(s)
        qo = 2 * s.batch * self.q_len * s.num_q_heads * s.head_dim * 2
        tables = int(sum(W.nblocks(int(L)) for L in self.lens)) * 4 + s.batch * 4
        return {"kv": kv, "q_out": qo, "tables": tables, "decode_total": kv + qo + tables}


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


def profiled_traffic(workload: str, kv_name: str) -> int | None:
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken from the current kernel source."""
    p = os.path.join(ROOT, "profiles", "decode_traffic_%s_%s.txt" % (workload, kv_name))
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if "=" in line and not line.startswith("#"):
            k, v = line.strip().split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_hash") != decode_source_hash():
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
    attention) over a bounded sample of the workload's sequences, with the
    sample's cache written by the oracle itself."""

    def __init__(self, s: W.Spec, nseq: int):
        import oracle
        self.oracle = oracle
        self.s = s
        lens = W.decode_lens(s)
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
        for i, b in enumerate(sample):
            nb = W.nblocks(int(lens[b]))
            self.bt[i, :nb] = np.arange(nxt, nxt + nb, dtype=np.int32)
            nxt += nb
            k, v = W.seq_kv(s, b)
            L = int(lens[b])
            step = s.chunk_tokens or L
            for c0 in range(0, L, step):
                c1 = min(L, c0 + step)
                oracle.kv_cache_write(self.c, k[c0:c1].contiguous(), v[c0:c1].contiguous(),
                                      W.slots_for(self.bt[i], c0, c1 - c0))
        self.q = W.query(s)[sample].contiguous()
        self.lens = lens[sample].astype(np.int32)
        self.sample = sample
        self.tokens = int(self.lens.sum())

    def step(self):
        self.oracle.paged_decode(self.c, self.q, self.bt, self.lens, W.softmax_scale(self.s))

    def describe(self, reps: int, per: float) -> str:
        return ("%d of %d sequences (%d tokens, lengths %d..%d); oracle decode (gather, dequantize, fp64 "
                "attention) timed %d times, %.3f s each" % (len(self.sample), self.s.batch, self.tokens,
                                                            int(self.lens.min()), int(self.lens.max()), reps, per))


def oracle_baseline(s: W.Spec, budget_s: float, nseq: int) -> dict:
    """cpu_baseline: the oracle as it stands, timed for about budget_s seconds."""
    o = OracleSample(s, nseq)
    t_total, reps = 0.0, 0
    while reps < 1 or (t_total < budget_s and reps < 100000):
        t0 = time.perf_counter()
        o.step()
        t_total += time.perf_counter() - t0
        reps += 1
    per = t_total / reps
    return {"value": o.tokens * per_token_bytes(s) / per / 1e9, "unit": UNIT, "cores": o.oracle.num_threads(),
            "kind": "oracle", "sample": o.describe(reps, per)}


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
        "config": config_dict(args, s, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.oracle.num_threads(), "kind": "oracle",
                         "sample": o.describe(args.steps, per)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(args, s: W.Spec, st: Setup | None) -> dict:
    d = {"workload": args.workload + ": " + DESCR[args.workload] + "; KV " + DT_LABEL[s.kv_dtype] +
         ("; step = append 1 token per sequence + paged decode" if args.q_len == 1 else
          "; step = append %d tokens per sequence + multi-query decode verifying them (speculative decoding)"
          % args.q_len), "batch": s.batch, "q_len": args.q_len,
         "num_q_heads": s.num_q_heads, "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim,
         "block_size": 16, "kv_dtype": DT_LABEL[s.kv_dtype], "split_blocks": args.split_blocks,
         "parallelism": "replicas (one independent batch per GPU)"}
    if st is not None:
        b = st.step_bytes()
        d["context_tokens"] = int(st.lens.sum())
        d["kv_bytes_per_step"] = b["kv"]
        d["l2"] = ("inputs larger than L2: %.0f MB of KV read per step vs 126 MB L2; no flush"
                   % (b["kv"] / 1e6)) if b["kv"] > 2 * L2_BYTES else \
            "KV smaller than L2 (%.1f MB): numbers include L2 hits" % (b["kv"] / 1e6)
    return d


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

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
    st = Setup(s, device, args.split_blocks, args.q_len)
    stream = torch.cuda.current_stream(device)

    for _ in range(max(args.warmup, 3)):
        st.write()
        st.decode()
    torch.cuda.synchronize(device)

    K = args.steps
    clocks = ClockSampler(local)
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
    value = b["kv"] * world / (ms_step * 1e-3) / 1e9
    tok_s = s.batch * args.q_len * world / (ms_step * 1e-3)
    peaks = measured_peaks()
    achieved = b["decode_total"] / (dec_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": profiled_traffic(args.workload, DT_LABEL[s.kv_dtype]),
                "kernel": "paged_decode_kernel", "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, "
                "a read+write copy)", "bytes_per_launch": b["decode_total"], "avg_launch_ms": dec_ms,
                "timing": "CUDA events around each decode call (per pass: decode kernel, merge kernel of long split pairs) over K further steps"}

    e2e = run_e2e(st, args, world) if not args.no_e2e else None

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline and args.q_len == 1:
            cpu = oracle_baseline(s, args.cpu_budget, args.ref_seqs)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if s.kv_dtype == W.DT_BF16 else ("fp16" if s.kv_dtype == W.DT_FP16 else
                                                             DT_LABEL[s.kv_dtype] + "->f16"),
            "data": "synthetic", "config": config_dict(args, s, st),
            "frac_of_hbm_peak": value / world / peaks["hbm_gbs"],
            "frac_of_8tbs_spec": value / world / 8000.0,
            "decode_tok_s_per_layer": tok_s,
            # the decode call alone (no cache write): B x q_len / t(decode)
            "decode_only_tok_s_per_layer": s.batch * args.q_len * world / (dec_ms * 1e-3),
            "decode_kernel_ms": dec_ms, "write_kernel_ms": wr_ms,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            # per step: cache write, then per decode pass the split decode and the merge kernel of
            # long split pairs (short ones are merged inside the decode)
            "gpu_launches": (1 + 2 * decode_passes(args.q_len, s.num_q_heads // s.num_kv_heads)) * K,
            "clocks": clocks.summary(),
        }
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
    ap.add_argument("--workload", choices=sorted(DESCR), default="llama8b")
    ap.add_argument("--kv-dtype", choices=sorted(KV_NAMES), default=None)
    ap.add_argument("--split-blocks", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None, help="first N sequences only (profiling subsets)")
    ap.add_argument("--pool-blocks", type=int, default=None, help="smaller block pool (profiling subsets)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle timing")
    ap.add_argument("--ref-seqs", type=int, default=None, help="sequences in the oracle sample")
    ap.add_argument("--op", choices=["decode", "copy_blocks", "swap", "prefill"], default="decode")
    ap.add_argument("--op-blocks", type=int, default=4096, help="blocks moved per step (--op copy_blocks|swap)")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per sequence and step (> 1: multi-query decode, speculative verification)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.ref_seqs is None:
        args.ref_seqs = {"tiny": 4, "llama8b": 64, "fp8": 32, "llama70b": 4, "fp4": 16}[args.workload]
    if args.impl == "reference":
        run_reference(args)
    elif args.op == "prefill":
        run_prefill(args)
    elif args.op != "decode":
        run_block_op(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
