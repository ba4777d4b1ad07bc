"""The decode kernels' bounded waits, made to run out on purpose.

Every wait of the decode on one of its asynchronous copies gives up after a
limit; pqkv_set_decode_wait_limit_ns shortens that limit (for later launches)
so that waits give up while their copies are still on the way. The decode must
then report PQKV_DEVERR_TIMEOUT, still let every copy in flight land before its
warps exit (no PQKV_DEVERR_DRAIN), leave the context usable, and the next call
with the normal limit on the same stream must match the oracle. No copy is
dropped or corrupted to cause the timeout: only the limit is short.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")


def _case(kv_dtype, seed):
    """64 sequences of 1-3k tokens (about 0.5 GB of bf16 KV, many copies in
    flight at once), 32 q / 8 KV heads, head_dim 128; K/V drawn on the GPU."""
    B, Hq, H, D = 64, 32, 8, 128
    rng = np.random.default_rng(seed)
    lens = rng.integers(1024, 3072, size=B).astype(np.int32)
    nblk = (lens + 15) // 16
    nb = int(nblk.sum()) + 16
    ids = rng.permutation(nb).astype(np.int32)
    bt = np.full((B, int(nblk.max())), -1, np.int32)
    pos = 0
    for b in range(B):
        bt[b, :nblk[b]] = ids[pos:pos + nblk[b]]
        pos += nblk[b]
    g = pq.allocate_cache(kv_dtype, nb, H, D, fill=0xFF)
    gen = torch.Generator(device="cuda").manual_seed(seed)
    err = gh.err_flag()
    kv = []
    for b in range(B):
        k = torch.randn((int(lens[b]), H, D), generator=gen, device="cuda").to(torch.bfloat16)
        v = torch.randn((int(lens[b]), H, D), generator=gen, device="cuda").to(torch.bfloat16)
        sl = np.arange(int(lens[b]))
        slots = (bt[b, sl // 16].astype(np.int64) * 16 + sl % 16).astype(np.int32)
        pq.kv_cache_write(k, v, torch.from_numpy(slots).cuda(), g, err)
        kv.append((k, v))
    q = torch.randn((B, Hq, D), generator=gen, device="cuda").to(torch.bfloat16)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return g, bt, lens, q, kv


def _oracle_check(g, bt, lens, q, kv, out, sample):
    """Oracle output of the sampled sequences (their K/V rewritten by the oracle
    into a compact pool) against the GPU output."""
    n = [int((lens[b] + 15) // 16) for b in sample]
    o = oracle.Cache(g.kv_dtype, sum(n), g.num_kv_heads, g.head_dim)
    obt = np.full((len(sample), max(n)), -1, np.int32)
    nxt = 0
    for i, b in enumerate(sample):
        obt[i, :n[i]] = np.arange(nxt, nxt + n[i])
        nxt += n[i]
        k, v = kv[b]
        assert oracle.kv_cache_write(o, k.cpu(), v.cpu(), np.arange(int(lens[b]), dtype=np.int32) + 16 * int(obt[i, 0])) == 0
    ref, oerr = oracle.paged_decode(o, q[sample].cpu(), obt, lens[sample], 1.0 / np.sqrt(g.head_dim))
    assert oerr == 0
    gh.assert_close(out[sample], ref, g.kv_dtype, tag="after a timeout")


@pytest.mark.parametrize("kv_dtype", [pq.BF16, pq.FP8_E4M3, pq.FP4_E2M1])
def test_decode_wait_limit_runs_out_and_the_next_call_is_correct(kv_dtype):
    """bf16 and FP8 warps wait on copies still on the way, so a 1 ns limit runs
    out; FP4 warps spend longer on each block than its next copies take to
    land, so their waits may all find the data there: for FP4 a timeout is
    checked when it happens, not required."""
    g, bt, lens, q, kv = _case(kv_dtype, seed=40 + kv_dtype)
    btd, sld = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    B, Hq, D = q.shape
    ws = pq.decode_workspace(B, Hq, g.num_kv_heads, D, bt.shape[1])
    out = torch.empty_like(q)
    scale = 1.0 / np.sqrt(D)
    seen = 0
    pq.set_decode_wait_limit_ns(1)
    try:
        for _ in range(5):
            err = gh.err_flag()
            pq.paged_decode_attention(q, g, btd, sld, scale, out, ws, err)
            torch.cuda.synchronize()  # the context is still usable: no fault, no hang
            e = int(err.item())
            assert e & pq.DEVERR_DRAIN == 0, "a copy was still in flight when its warp gave up draining"
            assert e & ~pq.DEVERR_TIMEOUT == 0
            seen += (e & pq.DEVERR_TIMEOUT) != 0
            if seen:
                break
    finally:
        pq.set_decode_wait_limit_ns(0)
    assert seen or kv_dtype == pq.FP4_E2M1, "no wait ran out with a 1 ns limit"
    # the next call with the normal limit, on the same stream
    err = gh.err_flag()
    pq.paged_decode_attention(q, g, btd, sld, scale, out, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.isfinite(out).all()
    _oracle_check(g, bt, lens, q, kv, out, [0, int(np.argmax(lens)), 37])
