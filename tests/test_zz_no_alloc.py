"""The decode entry point for callers that cannot allocate device memory
(pqkv_paged_decode_attention_noalloc: its scratch is a static device array
inside the library), called through the C ABI, against the regular entry point
that takes a caller-allocated workspace. Two calls in a row with different
inputs: the second must not see anything left in the shared scratch by the
first. Collected last so that a run stopping at the first failure has already
run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from tests import gpu_helpers as gh
from tests.helpers import random_tables, slots

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")


def _make(kv_dtype, qdt, lens, Hq, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    nb = sum((L + 15) // 16 for L in lens) + 5
    bt = random_tables(rng, lens, nb)
    g = pq.allocate_cache(kv_dtype, nb, Hkv, D, fill=0xFF)
    e = gh.err_flag()
    for b, L in enumerate(lens):
        k = torch.from_numpy(rng.standard_normal((L, Hkv, D)).astype(np.float32)).to(qdt).cuda()
        v = torch.from_numpy(rng.standard_normal((L, Hkv, D)).astype(np.float32)).to(qdt).cuda()
        pq.kv_cache_write(k, v, torch.from_numpy(slots(bt[b], 0, L)).cuda(), g, e)
    q = torch.from_numpy(rng.standard_normal((len(lens), Hq, D)).astype(np.float32)).to(qdt).cuda()
    torch.cuda.synchronize()
    assert int(e.item()) == 0
    return g, torch.from_numpy(bt).cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), q


def _noalloc(g, bt, sl, q, scale, split=0):
    out = torch.empty_like(q)
    err = gh.err_flag()
    ptr = lambda t: None if t is None else t.data_ptr()
    rc = pq.lib().pqkv_paged_decode_attention_noalloc(
        ptr(q), pq.BF16 if q.dtype == torch.bfloat16 else pq.FP16, q.shape[0], q.shape[1], ptr(g.cache),
        ptr(g.scales), ptr(g.outliers_idx), ptr(g.outliers_val), g.kv_dtype, g.num_blocks, g.num_kv_heads,
        g.head_dim, ptr(bt), bt.shape[1], ptr(sl), ctypes.c_float(scale), split, ptr(out), ptr(err),
        torch.cuda.current_stream().cuda_stream)
    return rc, out, err


def _regular(g, bt, sl, q, scale, split=0):
    out = torch.empty_like(q)
    err = gh.err_flag()
    ws = pq.decode_workspace(q.shape[0], q.shape[1], g.num_kv_heads, g.head_dim, bt.shape[1], split)
    pq.paged_decode_attention(q, g, bt, sl, scale, out, ws, err, split_blocks=split)
    return out, err


@pytest.mark.parametrize("kv_dtype", [pq.BF16, pq.FP8_E4M3])
def test_noalloc_matches_the_workspace_entry_point_twice_in_a_row(kv_dtype):
    qdt = torch.bfloat16
    first = _make(kv_dtype, qdt, [700, 3, 2100, 129], 32, 8, 128, seed=1)
    second = _make(kv_dtype, qdt, [17, 1500, 64, 900, 2], 32, 8, 128, seed=2)
    atol, rtol = gh.TOL[kv_dtype]
    for (g, bt, sl, q), scale in ((first, 0.088), (second, 0.1)):
        rc, out, err = _noalloc(g, bt, sl, q, scale)
        ref, rerr = _regular(g, bt, sl, q, scale)
        torch.cuda.synchronize()
        assert rc == pq.OK
        assert int(err.item()) == 0 and int(rerr.item()) == 0
        assert torch.isfinite(out).all()
        assert torch.allclose(out.float(), ref.float(), atol=atol, rtol=rtol)


def test_noalloc_rejects_requests_beyond_its_scratch():
    g, bt, sl, q = _make(pq.BF16, torch.bfloat16, [40, 20], 32, 8, 128, seed=3)
    need = pq.decode_workspace_bytes(2, 32, 8, 128, 1 << 16, 1)
    assert need > pq.NOALLOC_SCRATCH_BYTES
    big_bt = torch.full((2, 1 << 16), -1, dtype=torch.int32, device="cuda")
    big_bt[:, : bt.shape[1]] = bt
    rc, _, err = _noalloc(g, big_bt, sl, q, 0.1, split=1)
    torch.cuda.synchronize()
    assert rc == pq.ERR_SCRATCH and int(err.item()) == 0
