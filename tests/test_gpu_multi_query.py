"""GPU parity of multi-query decode (speculative verification: "vLLM" glossary,
"Speculative decoding") against the oracle: each sequence's last q_len
positions attend causally, which is the oracle's chunked prefill with chunks
of q_len tokens. The decode kernels put the q_len x G query rows of a KV head in
the columns of one or two 8-column tensor-core tiles (several passes when
q_len x G > 16); q_len = 1 must reproduce pqkv_paged_decode_attention bit for
bit."""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh
from tests.helpers import random_tables, slots

pytestmark = pytest.mark.gpu

pq = pytest.importorskip("paged_quantized_kv_cache_b200")

CASES = [
    # kv_dtype, q dtype, D, Hq, Hkv, q_len, split_blocks
    (pq.BF16, torch.bfloat16, 128, 32, 8, 2, 0),
    (pq.FP16, torch.float16, 64, 8, 8, 8, 0),
    (pq.FP8_E4M3, torch.bfloat16, 128, 32, 8, 2, 0),
    (pq.FP8_E4M3, torch.bfloat16, 128, 32, 8, 2, 3),
    (pq.FP8_E5M2, torch.float16, 64, 16, 8, 4, 0),
    (pq.FP4_E2M1, torch.bfloat16, 128, 32, 8, 2, 0),
    (pq.FP4_E2M1, torch.float16, 64, 8, 4, 3, 2),
    # 9..16 query rows per KV head: one pass with two column tiles
    (pq.BF16, torch.bfloat16, 128, 32, 8, 4, 0),
    (pq.FP16, torch.float16, 64, 8, 8, 16, 0),
    (pq.BF16, torch.bfloat16, 128, 24, 8, 5, 2),     # G = 3: 15 rows, the second tile part-filled
    (pq.FP8_E5M2, torch.float16, 64, 16, 8, 8, 0),
    (pq.FP4_E2M1, torch.bfloat16, 128, 32, 8, 4, 0),
    (pq.FP4_E2M1, torch.float16, 64, 32, 4, 2, 2),
    # more rows than two tiles hold: several passes over the KV, the last one narrower
    (pq.FP8_E4M3, torch.bfloat16, 128, 32, 8, 5, 3),
    (pq.FP4_E2M1, torch.bfloat16, 64, 32, 4, 3, 0),
    (pq.BF16, torch.bfloat16, 128, 32, 8, 11, 0),
]


def _build(kv_dtype, qdt, D, Hq, Hkv, k, lens, seed):
    rng = np.random.default_rng(seed)
    nb = sum((L + 15) // 16 for L in lens) + 5
    bt = random_tables(rng, lens, nb)
    g, o = gh.new_pair(kv_dtype, nb, Hkv, D)
    in_dt = torch.float16 if qdt == torch.float16 else torch.bfloat16
    for b, L in enumerate(lens):
        if L == 0:
            continue
        kk = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        vv = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        if kv_dtype == pq.FP4_E2M1:
            for h in range(Hkv):
                kk[:, h, rng.choice(D, 2, replace=False)] *= 16
                vv[:, h, rng.choice(D, 2, replace=False)] *= 16
        ge, oe = gh.write_both(g, o, torch.from_numpy(kk).to(in_dt), torch.from_numpy(vv).to(in_dt),
                               slots(bt[b], 0, L))
        assert ge == oe == 0
    q = torch.from_numpy(rng.standard_normal((len(lens), k, Hq, D)).astype(np.float32)).to(qdt)
    return g, o, bt, q


def _mq(g, q, bt, lens, scale, split=0):
    B, k, Hq, D = q.shape
    out = torch.full_like(q.cuda(), float("nan"))
    ws = pq.multi_query_decode_workspace(B, k, Hq, g.num_kv_heads, D, bt.shape[1], split)
    ws.fill_(0xAB)
    e = gh.err_flag()
    pq.paged_multi_query_decode_attention(q.cuda(), g, torch.from_numpy(np.ascontiguousarray(bt, np.int32)).cuda(),
                                          torch.from_numpy(np.array(lens, np.int32)).cuda(), scale, out, ws, e,
                                          split_blocks=split)
    torch.cuda.synchronize()
    return out, int(e.item())


@pytest.mark.parametrize("case", CASES, ids=lambda c: "kv%d-D%d-G%d-k%d-s%d" % (c[0], c[2], c[3] // c[4], c[5], c[6]))
def test_multi_query_decode_matches_oracle(case):
    kv_dtype, qdt, D, Hq, Hkv, k, split = case
    lens = [max(L, k) for L in (37, 200, 16, 1000, 9)]  # each sequence holds its q_len query tokens
    g, o, bt, q = _build(kv_dtype, qdt, D, Hq, Hkv, k, lens, seed=70 + kv_dtype + k)
    scale = 1.0 / np.sqrt(D)
    out, err = _mq(g, q, bt, lens, scale, split)
    cu = np.arange(0, (len(lens) + 1) * k, k, dtype=np.int32)
    ref, rerr = oracle.paged_prefill(o, q.reshape(-1, Hq, D), cu, bt, np.array(lens, np.int32), scale)
    assert err == rerr == 0
    gh.assert_close(out.reshape(-1, Hq, D), ref, kv_dtype, tag="multi-query")


@pytest.mark.parametrize("kv_dtype,qdt", [(pq.BF16, torch.bfloat16), (pq.FP8_E4M3, torch.bfloat16),
                                          (pq.FP4_E2M1, torch.bfloat16)])
def test_one_query_token_is_plain_decode_bit_for_bit(kv_dtype, qdt):
    lens = [300, 45, 1024]
    g, o, bt, q = _build(kv_dtype, qdt, 128, 32, 8, 1, lens, seed=80)
    a, ea = _mq(g, q, bt, lens, 0.09)
    b, eb = gh.decode_gpu(g, q[:, 0], bt, np.array(lens, np.int32), 0.09)
    assert ea == eb == 0
    assert torch.equal(a[:, 0], b)


def test_sequence_shorter_than_its_query_tokens_and_limits():
    kv_dtype, qdt, D, Hq, Hkv, k = pq.FP16, torch.float16, 64, 8, 4, 4
    lens = [40, 3, 0, 17]
    g, o, bt, q = _build(kv_dtype, qdt, D, Hq, Hkv, k, lens, seed=81)
    out, err = _mq(g, q, bt, lens, 0.125)
    assert err == pq.DEVERR_SEQ_LEN
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)
    keep = [0, 3]
    ref, _ = oracle.paged_prefill(o, q[keep].reshape(-1, Hq, D), np.arange(0, 3 * k, k, dtype=np.int32),
                                  bt[keep], np.array([lens[i] for i in keep], np.int32), 0.125)
    gh.assert_close(out[keep].reshape(-1, Hq, D), ref, kv_dtype, tag="valid sequences")
    # more than 64 query tokens, or a workspace sized for too few columns, is
    # rejected before anything runs
    ws = pq.multi_query_decode_workspace(1, 4, 8, 4, 64, bt.shape[1])
    for kq, w in ((65, ws), (4, ws[:16])):
        big = torch.zeros((1, kq, 8, 64), dtype=torch.float16, device="cuda")
        with pytest.raises(pq.PqkvError):
            pq.paged_multi_query_decode_attention(big, g, torch.from_numpy(bt[:1].copy()).cuda(),
                                                  torch.tensor([100], dtype=torch.int32, device="cuda"), 0.1,
                                                  torch.empty_like(big), w, gh.err_flag())
