"""The FP4 cache write against the oracle on every (input value, group scale)
pair that can occur together ("vLLM 0.7 Ships Unified KV Cache Compression",
"Technical Breakdown", step 3: each 16-channel group of a token is normalized by
its E4M3 scale = e4m3(absmax / 6) and rounded to E2M1).

For each positive finite E4M3 scale code sc, the group absmax a is the largest
input value whose scale is sc (capped where the quotient saturates anyway), and
the other members of the group run over every input value of magnitude <= a,
both signs, zeros and subnormals included: that is every input x that can be
divided by that scale. Each block plants one x16 outlier channel (channel 0 of
token 0) so that the outlier set is that one channel. Blocks whose channel
norms span many binades take the write's channel-order statistics, the others
its tree of exact partial sums; both must give the oracle's outlier set. Every
byte of the cache (codes, scales, outlier indices and values) must match the
oracle, for bf16 and fp16 inputs and head dims 128 and 64, K and V layouts.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")


def _finite_values(dt):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(dt)
    v = t.float().numpy()
    return np.unique(v[np.isfinite(v)])


def _scale_code(a):
    """E4M3 code of RN32(a / 6), saturating (a >= 0)."""
    y = (a.astype(np.float32) / np.float32(6.0)).astype(np.float32)
    y = np.minimum(y, np.float32(448.0))
    return torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _build_tokens(dt, D):
    """Tokens [T][D] (float32 values exactly representable in dt) grouped in
    16-token blocks, each block on one scale code."""
    vals = _finite_values(dt)
    pos = vals[vals > 0]
    codes = _scale_code(pos)
    e4m3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    G = D // 16
    per_token = (G - 1) * 15 + 14  # group 0 keeps channel 0 for the outlier and channel 1 for a
    blocks = []
    for sc in range(1, 127):
        have = pos[codes == sc]
        if have.size == 0:
            continue
        a = float(have.max())
        sd = float(e4m3[sc])
        if a > 8 * sd:  # beyond 8 x scale every quotient saturates to 6: cap
            a = float(vals[vals <= 8 * sd].max())
            if _scale_code(np.array([a], np.float32))[0] != sc:
                continue
        mem = vals[np.abs(vals) <= a]
        mem = np.concatenate([mem, [-0.0]])
        ntok = -(-mem.size // per_token)
        ntok = -(-ntok // 16) * 16
        m = np.zeros(ntok * per_token, np.float32)
        m[:mem.size] = mem
        m = m.reshape(ntok, per_token)
        tok = np.zeros((ntok, D), np.float32)
        tok[:, 1] = a
        tok[:, 2:16] = m[:, :14]
        for g in range(1, G):
            tok[:, 16 * g] = a
            tok[:, 16 * g + 1:16 * g + 16] = m[:, 14 + 15 * (g - 1):14 + 15 * g]
        big = min(16.0 * a, float(vals.max()))
        tok[0::16, 0] = big  # one outlier channel per block
        blocks.append(tok)
    return np.concatenate(blocks)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("D", [128, 64])
def test_fp4_write_matches_the_oracle_on_every_value_and_scale(dt, D):
    x = _build_tokens(dt, D)
    T = x.shape[0]
    nb = T // 16
    t = torch.from_numpy(x).to(dt)[:, None, :].contiguous()
    assert torch.equal(t.float()[:, 0, :], torch.from_numpy(x))  # exact in the input type
    g, o = gh.new_pair(pq.FP4_E2M1, nb, 1, D)
    slots = np.arange(T, dtype=np.int32)
    ge, oe = gh.write_both(g, o, t, t, slots)
    assert ge == 0 and oe == 0
    gh.assert_cache_equal(g, o, tag="fp4 exhaustive %s D%d" % (dt, D))
    # the planted channel is the outlier of most blocks
    idx = o.oidx.reshape(nb, 1, 2, 8)[:, 0, :, 0]
    assert (idx == 0).mean() > 0.9
