"""Host-side logic of bench.py that needs no GPU: the output-error statistics
against the oracle, the outlier-selection counts of the FP4 workload, the shared
config keys of both arms and the byte counts of the write and decode lines."""
import types

import numpy as np
import torch

import bench
import oracle
import workloads as W


def test_oracle_error_statistics():
    s = bench.bench_spec("tiny", None)
    o = bench.OracleSample(s, 4)
    ref = o.step()
    full = torch.zeros((s.batch, s.num_q_heads, s.head_dim), dtype=torch.float64)
    full[o.sample] = torch.from_numpy(ref)
    e = o.errors(full)
    assert e["max_abs_err"] == 0.0 and e["tol_used"] == 0.0
    bumped = full.clone()
    bumped[o.sample[0], 0, 0] += 0.01  # beyond 2e-3 + 1e-2 |ref| unless |ref| > 0.8
    e = o.errors(bumped)
    assert abs(e["max_abs_err"] - 0.01) < 1e-12
    assert abs(e["tol_used"] - 0.01 / (2e-3 + 1e-2 * abs(ref[0, 0, 0]))) < 1e-9


def test_oracle_sample_writes_like_the_bench():
    """The sample's cache takes the prefill and then the appended token as two
    calls; for FP8 that differs from one call when the token grows the scale."""
    s = bench.bench_spec("tiny", "fp8_e4m3")
    s.q_dtype = W.DT_BF16
    o = bench.OracleSample(s, 4)
    lens0 = W.seq_lens(s)
    c2 = oracle.Cache(s.kv_dtype, o.c.nb, s.num_kv_heads, s.head_dim)
    for i, b in enumerate(o.sample):
        k, v = W.seq_kv(s, b)
        L0, L = int(lens0[b]), int(o.lens[i])
        oracle.kv_cache_write(c2, k[:L0].contiguous(), v[:L0].contiguous(), W.slots_for(o.bt[i], 0, L0))
        oracle.kv_cache_write(c2, k[L0:L].contiguous(), v[L0:L].contiguous(), W.slots_for(o.bt[i], L0, L - L0))
    for a, b in zip(o.c.arrays(), c2.arrays()):
        if a is not None:
            np.testing.assert_array_equal(a, b)


def test_fp4_outlier_counts():
    s = W.spec("fp4", batch=2)
    H = s.num_kv_heads
    lens0 = W.seq_lens(s)
    nfull = [int(L) // 16 for L in lens0]
    nb = sum(nfull) + 8
    bt = np.full((2, max(nfull) + 1), -1, np.int32)
    bt[0, :nfull[0]] = np.arange(nfull[0])
    bt[1, :nfull[1]] = np.arange(nfull[0], nfull[0] + nfull[1])
    planted = W.outlier_channels(s)
    idx = np.full((nb, H, 2, 8), 0xFF, np.uint8)
    idx[:, :, :, 0] = planted[None, :, :, 0]
    idx[:, :, :, 1] = planted[None, :, :, 1]
    # one extra channel in one (block, head, K|V); one planted channel missing in another
    extra_ch = next(c for c in range(128) if c not in planted[3, 1])
    idx[5, 3, 1, :3] = np.sort([planted[3, 1, 0], planted[3, 1, 1], extra_ch])
    idx[7, 0, 0, 1] = 0xFF
    st = types.SimpleNamespace(s=s, tab=types.SimpleNamespace(num_blocks=nb, block_tables=bt),
                               cache=types.SimpleNamespace(outliers_idx=torch.from_numpy(idx.reshape(-1))))
    r = bench.fp4_outlier_stats(st)
    n = (nfull[0] + nfull[1]) * H * 2
    assert r["blocks_checked"] == n
    assert r["exact"] == n - 2
    assert r["with_false_positives"] == 1 and r["false_positive_channels"] == 1
    assert r["missed_planted"] == 1


def test_config_keys_and_byte_counts():
    args = types.SimpleNamespace(workload="llama70b", q_len=1, split_blocks=32)
    s = bench.bench_spec("llama70b", None)
    d = bench.config_dict(args, s)
    for k in ("context_tokens", "kv_bytes_per_step", "l2", "split_blocks", "kv_dtype"):
        assert k in d
    # unique tokens: sequences 1-3 reuse sequence 0's 4096-token prefix
    lens = W.decode_lens(s)
    assert bench.unique_tokens(s) == int(lens.sum()) - 3 * 4096
    assert d["kv_bytes_per_step"] == bench.unique_tokens(s) * 8 * 2 * 128 * 2
    s8 = bench.bench_spec("llama70b", "fp8_e4m3")
    assert bench.per_token_bytes(s8) == 8 * 2 * 128 + 8  # codes + the 16-byte scale granule per block / 16
    # the FP4 chunk write of 512 tokens x 256 sequences: about 705 MB
    b = bench.write_call_bytes(W.DT_FP4, 131072, 8, 128, 131072 // 16)
    assert 700e6 < b < 710e6


def test_profiled_traffic_only_for_its_source_split_and_query_length(tmp_path, monkeypatch):
    """A committed ncu traffic figure is used only while it describes the kernel
    being timed: same decode source, same split, one query token per sequence."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = "# comment\nsource_hash=%s\nsplit_blocks=32\ndram_bytes_per_launch=123456\n" % bench.decode_source_hash()
    (prof / "decode_traffic_llama70b_bf16.txt").write_text(good)
    (prof / "decode_traffic_llama70b_fp8_e4m3.txt").write_text(good.replace(bench.decode_source_hash(), "0" * 16))
    h = bench.decode_source_hash()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "decode_source_hash", lambda: h)
    assert bench.profiled_traffic("llama70b", "bf16", 32) == 123456
    assert bench.profiled_traffic("llama70b", "bf16", 0) is None        # another split
    assert bench.profiled_traffic("llama70b", "bf16", 32, q_len=4) is None  # multi-query decode
    assert bench.profiled_traffic("llama70b", "fp8_e4m3", 32) is None   # taken from another source
    assert bench.profiled_traffic("llama8b", "bf16", 32) is None        # no capture
