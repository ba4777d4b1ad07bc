"""Why the decode does not compute P.V as a block-scaled tensor-core product.

A block-scaled product (both operands in 8-bit or smaller codes, with a
power-of-two scale per 32 elements along the contraction) would need V stored
as E2M1 codes grouped along tokens and the probabilities P rounded to E4M3 per
32 tokens ("vLLM" glossary, "Speculative decoding": several query tokens would
fill the product's N dimension). This measures, on a sequence of the fp4
workload (its planted x16 outlier channels kept in fp16 as in the cache), what
rounding P to E4M3 alone does to the output, with V already in that layout and
the scale of each 32-token group the smallest power of two that avoids
clipping (the most favourable choice): the error is many times the tolerance
the 4-bit path is held to (5e-3 + 1e-2 |ref|), so such a variant could not
match an oracle of its own format. It also measures V grouped along tokens
against the layout the cache uses (E4M3 scale per 16 channels of one token),
both against the unquantized values: the token grouping is the less accurate.
"""
import numpy as np
import torch

import oracle
import workloads as W

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e2m1(x):
    """Nearest E2M1 value (OCP Microscaling Formats), magnitude clipped at 6."""
    a = np.minimum(np.abs(x), 6.0)
    return np.sign(x) * E2M1[np.abs(a[..., None] - E2M1).argmin(-1)]


def _e4m3(x):
    return torch.from_numpy(np.clip(x, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _pow2_scale(amax, fmax):
    """Smallest power of two X with amax / X <= fmax (1 for an all-zero group)."""
    return np.where(amax > 0, 2.0 ** np.ceil(np.log2(np.maximum(amax, 1e-300) / fmax)), 1.0)


def _group_along_tokens(x, n, quant, fmax):
    """x [L][C] quantized in groups of n consecutive tokens per column."""
    L = x.shape[0]
    Lp = -(-L // n) * n
    xp = np.zeros((Lp,) + x.shape[1:])
    xp[:L] = x
    g = xp.reshape((Lp // n, n) + x.shape[1:])
    X = _pow2_scale(np.abs(g).max(1, keepdims=True), fmax)
    return (quant(g / X) * X).reshape(xp.shape)[:L]


def test_p_in_e4m3_exceeds_the_fp4_tolerance():
    s = W.spec("fp4")
    s.append_tokens = 0
    lens = W.seq_lens(s)
    b = int(np.argsort(lens)[len(lens) // 4])  # a sequence of about 3k tokens
    L = int(lens[b])
    k, v = W.seq_kv(s, b, with_append=False)
    c = oracle.Cache(W.DT_FP4, (L + 15) // 16, s.num_kv_heads, s.head_dim)
    bt = np.arange((L + 15) // 16, dtype=np.int32)
    for c0 in range(0, L, 512):  # the workload's 512-token chunked writes
        c1 = min(L, c0 + 512)
        oracle.kv_cache_write(c, k[c0:c1].contiguous(), v[c0:c1].contiguous(), W.slots_for(bt, c0, c1 - c0))
    q = W.query(s)[b].double().numpy()
    G = s.num_q_heads // s.num_kv_heads
    worst_p, worst_new, worst_cur = 0.0, 0.0, 0.0
    for h in range(s.num_kv_heads):
        kd, vd, _ = oracle.gather(c, bt, L, h)
        vx = v[:, h].double().numpy()
        vq = _group_along_tokens(vx, 32, _e2m1, 6.0)
        oidx = c.oidx.reshape(-1, s.num_kv_heads, 2, 8)[:, h, 1, :4]
        for blk in range(len(bt)):  # outlier channels stay exact fp16, as in the cache
            for ch in oidx[blk]:
                if ch != 0xFF:
                    vq[16 * blk:16 * blk + 16, ch] = vd[16 * blk:16 * blk + 16, ch]
        for hq in range(G * h, G * h + G):
            sc = W.softmax_scale(s) * (kd @ q[hq])
            p = np.exp(sc - sc.max())
            pq = _group_along_tokens(p[:, None], 32, _e4m3, 448.0)[:, 0]
            exact_p = (p @ vq) / p.sum()
            tol = lambda d, ref: float((np.abs(d) / (5e-3 + 1e-2 * np.abs(ref))).max())  # noqa: E731
            worst_p = max(worst_p, tol((pq @ vq) / p.sum() - exact_p, exact_p))
            unq = (p @ vx) / p.sum()
            worst_new = max(worst_new, tol(exact_p - unq, unq))
            worst_cur = max(worst_cur, tol((p @ vd) / p.sum() - unq, unq))
    print("tolerance units: P in E4M3 %.1f; V along tokens vs unquantized %.1f; cache layout %.1f"
          % (worst_p, worst_new, worst_cur))
    assert worst_p > 2.0  # beyond the tolerance (1.0), by a wide margin
    assert worst_new > worst_cur
