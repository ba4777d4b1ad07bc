"""bf16 queries outside the f16 range, with FP8 and FP4 caches.

The tensor-core products of quantized caches take f16 operands, so a bf16
query is narrowed to f16. Each query row is first scaled by a power of two that
brings its largest |q| to [2^13, 2^14), and the logits are scaled back, so
that neither |q| above the f16 maximum (65504) nor |q| below the smallest f16
normal (2^-14) changes the result. Checked on decode, multi-query decode and
chunked prefill: q x 2^17 (up to about 5e5) and q x 2^-20 (about 1e-6), with
the softmax scale divided by the same factor, must give the very outputs of
the unscaled call, and match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh
from tests.test_gpu_parity import _scenario

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")

CASES = [
    (pq.FP8_E4M3, torch.bfloat16, 128, 32, 8),
    (pq.FP8_E5M2, torch.bfloat16, 64, 16, 2),
    (pq.FP4_E2M1, torch.bfloat16, 128, 32, 8),
]


def _decode(g, q, bt, lens, scale, q_len=1):
    B = len(lens)
    btd = torch.from_numpy(np.ascontiguousarray(bt)).cuda()
    sl = torch.from_numpy(np.array(lens, np.int32)).cuda()
    out = torch.empty_like(q.cuda())
    err = gh.err_flag()
    if q_len == 1:
        ws = pq.decode_workspace(B, q.shape[1], g.num_kv_heads, g.head_dim, bt.shape[1])
        pq.paged_decode_attention(q.cuda(), g, btd, sl, scale, out, ws, err)
    else:
        ws = pq.multi_query_decode_workspace(B, q_len, q.shape[2], g.num_kv_heads, g.head_dim, bt.shape[1])
        pq.paged_multi_query_decode_attention(q.cuda(), g, btd, sl, scale, out, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out


def _prefill(g, q, bt, lens, scale, qn):
    B = len(lens)
    cu = torch.arange(0, (B + 1) * qn, qn, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q.cuda())
    err = gh.err_flag()
    pq.paged_prefill_attention(q.cuda(), cu, qn, g, torch.from_numpy(np.ascontiguousarray(bt)).cuda(),
                               torch.from_numpy(np.array(lens, np.int32)).cuda(), scale, out, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-D%d" % (pq.DTYPE_NAMES[c[0]], c[2]))
@pytest.mark.parametrize("power", [17, -20])
def test_query_scaled_beyond_the_f16_range(case, power):
    lens = [17, 100, 513, 1000]
    g, o, bt, q = _scenario(case, lens, seed=300 + case[0])
    scale = float(np.float32(1.0 / np.sqrt(case[2])))
    f = 2.0 ** power
    qs = (q.float() * f).to(torch.bfloat16)
    assert torch.equal(qs.float(), q.float() * f)  # a power of two: exact in bf16
    ss = float(np.float32(scale / f))
    base = _decode(g, q, bt, lens, scale)
    got = _decode(g, qs, bt, lens, ss)
    assert torch.equal(got, base)
    ref, oerr = oracle.paged_decode(o, qs, bt, np.array(lens, np.int32), ss)
    assert oerr == 0
    gh.assert_close(got, ref, case[0], tag="q x 2^%d" % power)
    # multi-query decode (3 query tokens per sequence)
    Hq, D = case[3], case[2]
    rng = np.random.default_rng(7)
    q3 = torch.from_numpy(rng.standard_normal((len(lens), 3, Hq, D)).astype(np.float32)).to(torch.bfloat16)
    q3s = (q3.float() * f).to(torch.bfloat16)
    base3 = _decode(g, q3, bt, lens, scale, q_len=3)
    got3 = _decode(g, q3s, bt, lens, ss, q_len=3)
    assert torch.equal(got3, base3)
    # chunked prefill (the last 16 positions of every sequence)
    q16 = torch.from_numpy(rng.standard_normal((len(lens) * 16, Hq, D)).astype(np.float32)).to(torch.bfloat16)
    q16s = (q16.float() * f).to(torch.bfloat16)
    basep = _prefill(g, q16, bt, lens, scale, 16)
    gotp = _prefill(g, q16s, bt, lens, ss, 16)
    assert torch.equal(gotp, basep)
    refp, oerr = oracle.paged_prefill(o, q16s, np.arange(0, 16 * (len(lens) + 1), 16, dtype=np.int32), bt,
                                      np.array(lens, np.int32), ss)
    assert oerr == 0
    gh.assert_close(gotp, refp, case[0], tag="prefill q x 2^%d" % power)
