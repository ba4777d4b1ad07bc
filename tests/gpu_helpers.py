"""Helpers for the GPU parity tests: drive the CUDA path (through the C ABI
binding) and the CPU oracle on the same seeded inputs and compare them."""
import json
import os

import numpy as np
import torch

import oracle
import paged_quantized_kv_cache_b200 as pq

# atol, rtol of attention outputs against the fp64 oracle
TOL = {pq.FP16: (2e-3, 1e-2), pq.BF16: (2e-3, 1e-2), pq.FP8_E4M3: (2e-3, 1e-2),
       pq.FP8_E5M2: (2e-3, 1e-2), pq.FP4_E2M1: (5e-3, 1e-2)}
POISON = 0xFF


def err_flag():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def new_pair(kv_dtype, nb, H, D):
    """A GPU cache and an oracle cache, both filled with the poison byte."""
    g = pq.allocate_cache(kv_dtype, nb, H, D, fill=POISON)
    o = oracle.Cache(kv_dtype, nb, H, D, poison=True)
    return g, o


def write_both(g, o, k, v, slots, expect_err=0):
    """One write call on both sides; returns (gpu_err, oracle_err)."""
    e = err_flag()
    pq.kv_cache_write(k.cuda(), v.cuda(), torch.from_numpy(np.ascontiguousarray(slots, np.int32)).cuda(), g, e)
    oe = oracle.kv_cache_write(o, k, v, slots)
    torch.cuda.synchronize()
    return int(e.item()), oe


def assert_cache_equal(g, o, block_ids=None, tag=""):
    """Bit-exact comparison of every cache array (all blocks, or block_ids)."""
    names = ("cache", "scales", "outliers_idx", "outliers_val")
    for name, ga, oa in zip(names, g.arrays(), o.arrays()):
        if ga is None:
            assert oa is None
            continue
        per_block = oa.size // o.nb
        gb = ga.view(o.nb, per_block)
        ob = oa.reshape(o.nb, per_block)
        if block_ids is not None:
            idx = torch.as_tensor(np.asarray(block_ids, np.int64), device="cuda")
            gb = gb.index_select(0, idx).cpu().numpy()
            ob = ob[np.asarray(block_ids)]
        else:
            gb = gb.cpu().numpy()
        if not np.array_equal(gb, ob):
            bad = np.argwhere(gb != ob)
            raise AssertionError("%s %s differs at %d bytes, first (block,byte)=%s gpu=%d oracle=%d" % (
                tag, name, len(bad), tuple(bad[0]), gb[tuple(bad[0])], ob[tuple(bad[0])]))


def decode_gpu(g, q, block_tables, seq_lens, scale, split_blocks=0):
    B, Hq, D = q.shape
    bt = torch.from_numpy(np.ascontiguousarray(block_tables, np.int32)).cuda()
    sl = torch.from_numpy(np.ascontiguousarray(seq_lens, np.int32)).cuda()
    out = torch.empty_like(q.cuda())
    ws = pq.decode_workspace(B, Hq, g.num_kv_heads, D, bt.shape[1], split_blocks)
    e = err_flag()
    pq.paged_decode_attention(q.cuda(), g, bt, sl, scale, out, ws, e, split_blocks=split_blocks)
    torch.cuda.synchronize()
    return out, int(e.item())


def _log_errors(tag, kv_dtype, d, ref, atol, rtol):
    """With PQKV_PARITY_LOG set, append the achieved error of one comparison to
    that file (JSON lines), so that the margin left under the tolerance is
    on record, not only pass / fail."""
    path = os.environ.get("PQKV_PARITY_LOG")
    if not path or d.size == 0:
        return
    rec = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "tag": tag,
           "kv_dtype": pq.DTYPE_NAMES.get(kv_dtype, str(kv_dtype)), "n": int(d.size),
           "max_abs_err": float(d.max()), "tol_used": float((d / (atol + rtol * np.abs(ref))).max()),
           "atol": atol, "rtol": rtol}
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def assert_close(out, ref, kv_dtype, tag=""):
    atol, rtol = TOL[kv_dtype]
    o = out.double().cpu().numpy()
    _log_errors(tag, kv_dtype, np.abs(o - ref), ref, atol, rtol)
    bad = ~(np.abs(o - ref) <= atol + rtol * np.abs(ref))
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError("%s: %d of %d outputs outside tolerance; first %s gpu=%r ref=%r" % (
            tag, int(bad.sum()), bad.size, i, o[i], ref[i]))
