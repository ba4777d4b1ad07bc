"""The decode entry point for callers that cannot allocate device memory
(pqkv_paged_decode_attention_noalloc: its scratch is a static device array
inside the library), called through the C ABI.

Callers such as a serving host whose device memory is all reserved by its own
pool, or a latency-critical path that may not call cudaMalloc (it can
synchronize the device), cannot pass a workspace. This entry point must give
the same results as the regular entry point that takes a caller-allocated
workspace, and as the CPU oracle, on consecutive calls whose sizes change (so
that the split-pair bookkeeping of one call lands where another call left
other bytes), and must not change the device memory in use.

Collected last so that a run stopping at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh
from tests.helpers import random_tables, slots

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")


def _make(kv_dtype, lens, Hq, Hkv, D, seed):
    """A GPU cache and an oracle cache with the same writes, and the query."""
    rng = np.random.default_rng(seed)
    nb = sum((L + 15) // 16 for L in lens) + 5
    bt = random_tables(rng, lens, nb)
    g, o = gh.new_pair(kv_dtype, nb, Hkv, D)
    for b, L in enumerate(lens):
        x = rng.standard_normal((2, L, Hkv, D)).astype(np.float32)
        if kv_dtype == pq.FP4_E2M1:
            x[:, :, :, 5] *= 16.0  # one outlier channel per head
        k = torch.from_numpy(x[0]).to(torch.bfloat16)
        v = torch.from_numpy(x[1]).to(torch.bfloat16)
        ge, oe = gh.write_both(g, o, k, v, slots(bt[b], 0, L))
        assert ge == 0 and oe == 0
    q = torch.from_numpy(rng.standard_normal((len(lens), Hq, D)).astype(np.float32)).to(torch.bfloat16)
    return g, o, bt, np.array(lens, np.int32), q


def _noalloc(g, bt, sl, q, scale, out, err, split=0):
    ptr = lambda t: None if t is None else t.data_ptr()
    return pq.lib().pqkv_paged_decode_attention_noalloc(
        ptr(q), pq.BF16, q.shape[0], q.shape[1], ptr(g.cache), ptr(g.scales), ptr(g.outliers_idx),
        ptr(g.outliers_val), g.kv_dtype, g.num_blocks, g.num_kv_heads, g.head_dim, ptr(bt), bt.shape[1], ptr(sl),
        ctypes.c_float(scale), split, ptr(out), ptr(err), torch.cuda.current_stream().cuda_stream)


def _regular(g, bt, sl, q, scale, split=0):
    out = torch.empty_like(q)
    err = gh.err_flag()
    ws = pq.decode_workspace(q.shape[0], q.shape[1], g.num_kv_heads, g.head_dim, bt.shape[1], split)
    pq.paged_decode_attention(q, g, bt, sl, scale, out, ws, err, split_blocks=split)
    return out, err


# (kv dtype, lengths, Hq, Hkv, head_dim, split_blocks): consecutive calls change
# the columns per KV head, the head size and the split, then repeat a layout
CALLS = [
    (pq.BF16, [700, 3, 2100, 129], 64, 8, 128, 0),
    (pq.BF16, [17, 1500, 64, 900, 2], 8, 8, 64, 0),
    (pq.FP8_E4M3, [300, 1200, 33], 32, 8, 128, 3),
    (pq.FP4_E2M1, [640, 77, 1999], 32, 8, 128, 0),
    (pq.BF16, [700, 3, 2100, 129], 64, 8, 128, 0),
    (pq.BF16, [1000, 50, 400, 1600], 64, 8, 128, 0),
]


def test_noalloc_matches_the_workspace_entry_point_and_the_oracle_over_changing_layouts():
    cases = [_make(kv, lens, Hq, Hkv, D, seed=10 + i) for i, (kv, lens, Hq, Hkv, D, _) in enumerate(CALLS)]
    dev = []
    for (g, o, bt, lens, q), call in zip(cases, CALLS):
        dev.append((torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), q.cuda(),
                    torch.empty((q.shape[0], q.shape[1], q.shape[2]), dtype=torch.bfloat16, device="cuda"),
                    gh.err_flag()))
    torch.cuda.synchronize()
    for i, ((g, o, bt, lens, q), (btd, sld, qd, out, err), call) in enumerate(zip(cases, dev, CALLS)):
        split = call[5]
        scale = 1.0 / np.sqrt(call[4])
        # the regular entry point first: it also loads the kernels this call uses
        ref, rerr = _regular(g, btd, sld, qd, scale, split)
        torch.cuda.synchronize()
        mem0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        rc = _noalloc(g, btd, sld, qd, scale, out, err, split)
        torch.cuda.synchronize()
        assert rc == pq.OK
        # nothing allocated: the first call in a process may load the library's
        # static array itself, every later one leaves device memory as it was
        assert torch.cuda.memory_allocated() == mem0
        if i > 0:
            assert torch.cuda.mem_get_info()[0] == free0
        assert int(err.item()) == 0 and int(rerr.item()) == 0
        assert torch.isfinite(out).all()
        atol, rtol = gh.TOL[g.kv_dtype]
        assert torch.allclose(out.float(), ref.float(), atol=atol, rtol=rtol)
        want, oerr = oracle.paged_decode(o, q, bt, lens, scale)
        assert oerr == 0
        gh.assert_close(out, want, g.kv_dtype, tag="no-alloc call %d" % i)


def test_noalloc_rejects_requests_beyond_its_scratch():
    g, _, bt, lens, q = _make(pq.BF16, [40, 20], 32, 8, 128, seed=3)
    need = pq.decode_workspace_bytes(2, 32, 8, 128, 1 << 16, 1)
    assert need > pq.NOALLOC_SCRATCH_BYTES
    big_bt = torch.full((2, 1 << 16), -1, dtype=torch.int32, device="cuda")
    big_bt[:, : bt.shape[1]] = torch.from_numpy(bt).cuda()
    out = torch.empty((2, 32, 128), dtype=torch.bfloat16, device="cuda")
    err = gh.err_flag()
    rc = _noalloc(g, big_bt, torch.from_numpy(lens).cuda(), q.cuda(), 0.1, out, err, split=1)
    torch.cuda.synchronize()
    assert rc == pq.ERR_SCRATCH and int(err.item()) == 0
