"""GPU parity at full size, in the launch configuration bench.py times, for the
multi-query decode step ("vLLM" glossary, "Speculative decoding"; bench.py
--q-len 2) and the chunked-prefill step ("Chunked prefill"; bench.py --op
prefill: 16 sequences, a U[0, 7680]-token prefix and a 512-token chunk each).

The oracle re-does the writes of a sample of sequences (shortest, longest and
a few more) in a compact pool; their cache bytes must match exactly and their
outputs within tolerance. Prefill rows are sampled too (first, last and some in
between); each sampled row is the oracle's decode at that row's position.
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


def _sample(s, n, seed=99):
    lens = W.decode_lens(s)
    order = [int(i) for i in np.argsort(lens, kind="stable")]
    rng = np.random.default_rng(seed)
    pick = {order[0], order[-1]}
    for b in rng.choice(s.batch, size=min(s.batch, n), replace=False):
        pick.add(int(b))
    return sorted(pick)


def _oracle_cache(s, st, sample, q_len):
    """Oracle cache of the sampled sequences after the same writes as the GPU
    (prefill in the workload's call sizes, then the step's q_len new tokens)."""
    tab = st.tab
    lens0, lens = W.seq_lens(s), W.decode_lens(s)
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
        step = s.chunk_tokens or L0
        for c0 in range(0, L0, max(1, step)):
            c1 = min(L0, c0 + step)
            assert oracle.kv_cache_write(o, k[c0:c1].contiguous(), v[c0:c1].contiguous(),
                                         W.slots_for(obt[i], c0, c1 - c0)) == 0
        newk.append(k[L0:L0 + q_len])
        newv.append(v[L0:L0 + q_len])
        newslots.append(W.slots_for(obt[i], L0, q_len))
    assert oracle.kv_cache_write(o, torch.cat(newk).contiguous(), torch.cat(newv).contiguous(),
                                 np.concatenate(newslots).astype(np.int32)) == 0
    for ga, oa in zip(st.cache.arrays(), o.arrays()):
        if ga is None:
            continue
        per = oa.size // len(gpu_ids)
        got = ga.view(tab.num_blocks, per).index_select(
            0, torch.as_tensor(gpu_ids, dtype=torch.int64, device="cuda")).cpu().numpy()
        assert np.array_equal(got, oa.reshape(len(gpu_ids), per))
    return o, obt


# q_len 2: one 8-column tile; 4: two tiles (G = 4); 8: two passes of two tiles
MQ = [("llama8b", None, 2), ("fp8", "fp8_e4m3", 2), ("fp4", None, 2),
      ("llama8b", None, 4), ("llama8b", None, 8), ("fp8", "fp8_e4m3", 4), ("fp4", None, 4)]


@pytest.mark.parametrize("name,kv,q_len", MQ, ids=["%s-%s-q%d" % (n, k or "default", q) for n, k, q in MQ])
def test_full_size_multi_query_decode(name, kv, q_len):
    s = bench.bench_spec(name, kv, q_len=q_len)
    st = bench.Setup(s, torch.device("cuda", 0), 0, q_len=q_len)
    st.write()
    st.decode()
    torch.cuda.synchronize()
    assert int(st.err.item()) == 0
    assert torch.isfinite(st.d_out).all()
    sample = _sample(s, 3)
    o, obt = _oracle_cache(s, st, sample, q_len)
    q = W.multi_query(s, q_len)[sample].contiguous()
    n = len(sample)
    lens = W.decode_lens(s)[sample].astype(np.int32)
    ref, oerr = oracle.paged_prefill(o, q.view(-1, s.num_q_heads, s.head_dim),
                                     np.arange(0, (n + 1) * q_len, q_len, dtype=np.int32), obt, lens,
                                     W.softmax_scale(s))
    assert oerr == 0
    gh.assert_close(st.d_out[sample].reshape(-1, s.num_q_heads, s.head_dim), ref, s.kv_dtype,
                    tag="%s q_len %d" % (name, q_len))


@pytest.mark.parametrize("kv", [None, "fp8_e4m3", "fp4"])
def test_full_size_chunked_prefill(kv):
    C = 512
    s = bench.bench_spec("prefill", kv, q_len=C)
    st = bench.Setup(s, torch.device("cuda", 0), 0, q_len=C, prefill=True)
    st.write()
    st.decode()
    torch.cuda.synchronize()
    assert int(st.err.item()) == 0
    assert torch.isfinite(st.d_out).all()
    sample = _sample(s, 2)
    o, obt = _oracle_cache(s, st, sample, C)
    rows = [0, 1, 31, 32, 200, 383, 510, 511]
    q = W.multi_query(s, C)[sample]
    lens = W.decode_lens(s)
    qs, tabs, ls, got = [], [], [], []
    for i, b in enumerate(sample):
        for r in rows:
            qs.append(q[i, r])
            tabs.append(obt[i])
            ls.append(int(lens[b]) - C + r + 1)  # the row's position + 1
            got.append(st.d_out[b, r])
    ref, oerr = oracle.paged_decode(o, torch.stack(qs).contiguous(), np.stack(tabs), np.array(ls, np.int32),
                                    W.softmax_scale(s))
    assert oerr == 0
    gh.assert_close(torch.stack(got), ref, s.kv_dtype, tag="prefill %s" % (kv or "bf16"))
