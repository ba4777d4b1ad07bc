"""GPU parity at the full sizes of the five workloads, in the launch
configuration bench.py times (its Setup: prefill written in the workload's
call sizes, then one step = append one token per sequence + paged decode).

The oracle re-does the same writes for a sample of sequences (shortest,
longest and a few in between, plus sequence 0 when a shared prefix is
sampled) in a compact pool; for those sequences every cache byte of every
block and every output must match (bytes exactly, outputs within tolerance).
For all sequences the outputs must be finite and no device error bit set.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gpu_helpers as gh

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
pq = pytest.importorskip("paged_quantized_kv_cache_b200")
bench = pytest.importorskip("bench")

CASES = [
    ("tiny", None, 0),
    ("llama8b", None, 0),
    ("fp8", "fp8_e4m3", 0),
    ("fp8", "fp8_e5m2", 0),
    ("llama70b", None, 32),
    ("llama70b", "fp8_e4m3", 32),
    ("llama70b", None, 0),
    ("llama70b", "fp8_e4m3", 0),
    ("fp4", None, 0),
]


def _sample(s, n):
    lens = W.decode_lens(s)
    order = [int(i) for i in np.argsort(lens, kind="stable")]
    rng = np.random.default_rng(99)
    pick = {order[0], order[-1]}
    for b in rng.choice(s.batch, size=min(s.batch, n), replace=False):
        pick.add(int(b))
    if s.shared_prefix_seqs and any(0 < b < s.shared_prefix_seqs for b in pick):
        pick.add(0)
    return sorted(pick)


@pytest.mark.parametrize("name,kv,split", CASES, ids=["%s-%s-split%d" % (c[0], c[1] or "default", c[2]) for c in CASES])
def test_full_size_workload(name, kv, split):
    s = bench.bench_spec(name, kv)
    st = bench.Setup(s, torch.device("cuda", 0), split)
    st.write()
    st.decode()
    torch.cuda.synchronize()
    assert int(st.err.item()) == 0
    out = st.d_out
    assert torch.isfinite(out).all()

    sample = _sample(s, 3 if s.batch > 4 else s.batch)
    tab = st.tab
    lens0 = W.seq_lens(s)
    lens = W.decode_lens(s)
    # compact oracle pool: GPU block id -> oracle block id
    gpu_ids = []
    for b in sample:
        for jj in range(W.nblocks(int(lens[b]))):
            bid = int(tab.block_tables[b, jj])
            if bid not in gpu_ids:
                gpu_ids.append(bid)
    remap = {g: i for i, g in enumerate(gpu_ids)}
    obt = np.full((len(sample), tab.max_blocks), -1, np.int32)
    for i, b in enumerate(sample):
        for jj in range(W.nblocks(int(lens[b]))):
            obt[i, jj] = remap[int(tab.block_tables[b, jj])]
    o = oracle.Cache(s.kv_dtype, len(gpu_ids), s.num_kv_heads, s.head_dim)
    in_dt = W.TORCH_DTYPE[W.input_dtype(s)]
    newk, newv, newslots = [], [], []
    for i, b in enumerate(sample):
        k, v = W.seq_kv(s, b)
        k, v = k.to(in_dt), v.to(in_dt)
        L0 = int(lens0[b])
        lo = s.shared_prefix_tokens if (0 < b < s.shared_prefix_seqs) else 0
        step = s.chunk_tokens or L0
        for c0 in range(lo, L0, step):
            c1 = min(L0, c0 + step)
            assert oracle.kv_cache_write(o, k[c0:c1].contiguous(), v[c0:c1].contiguous(),
                                         W.slots_for(obt[i], c0, c1 - c0)) == 0
        newk.append(k[L0:L0 + 1])
        newv.append(v[L0:L0 + 1])
        newslots.append(W.slots_for(obt[i], L0, 1)[0])
    assert oracle.kv_cache_write(o, torch.cat(newk).contiguous(), torch.cat(newv).contiguous(),
                                 np.array(newslots, np.int32)) == 0
    # every byte of the sampled sequences' blocks
    for ga, oa in zip(st.cache.arrays(), o.arrays()):
        if ga is None:
            continue
        per = oa.size // len(gpu_ids)
        got = ga.view(tab.num_blocks, per).index_select(
            0, torch.as_tensor(gpu_ids, dtype=torch.int64, device="cuda")).cpu().numpy()
        assert np.array_equal(got, oa.reshape(len(gpu_ids), per))
    q = W.query(s)[sample].contiguous()
    ref, oerr = oracle.paged_decode(o, q, obt, lens[sample].astype(np.int32), W.softmax_scale(s))
    assert oerr == 0
    gh.assert_close(out[sample], ref, s.kv_dtype, tag="%s %s" % (name, kv))
