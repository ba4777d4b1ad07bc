"""Shared helpers for the tests: small paged-cache scenarios built from seeded
random numbers, and brute-force references written from the definitions."""
import math

import numpy as np
import torch

BLOCK = 16


def random_tables(rng, lens, nb, max_blocks=None, shared_prefix_blocks=0, n_share=0):
    """Block tables with ids sampled without replacement from a pool of nb.
    Sequences 0..n_share-1 share their first shared_prefix_blocks ids."""
    nblk = [(int(L) + BLOCK - 1) // BLOCK for L in lens]
    if max_blocks is None:
        max_blocks = max(1, max(nblk))
    need = sum(nblk) - shared_prefix_blocks * max(0, n_share - 1)
    ids = rng.choice(nb, size=need, replace=False)
    bt = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    pos = 0
    prefix = None
    for b, n in enumerate(nblk):
        j0 = 0
        if b < n_share and shared_prefix_blocks:
            if prefix is None:
                prefix = ids[pos:pos + shared_prefix_blocks]
                pos += shared_prefix_blocks
            bt[b, :shared_prefix_blocks] = prefix
            j0 = shared_prefix_blocks
        bt[b, j0:n] = ids[pos:pos + n - j0]
        pos += n - j0
    return bt


def slots(bt_row, start, n):
    pos = np.arange(start, start + n)
    return (bt_row[pos // BLOCK].astype(np.int64) * BLOCK + pos % BLOCK).astype(np.int32)


def to_f64(t):
    return t.to(torch.float64).numpy()


def brute_force_attention(q, k, v, scale):
    """softmax(scale q.k) v with Python floats and math.fsum; q [D], k/v [L][D]."""
    L, D = len(k), len(q)
    s = [scale * math.fsum(q[c] * k[t][c] for c in range(D)) for t in range(L)]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    den = math.fsum(w)
    return [math.fsum(w[t] * v[t][c] for t in range(L)) / den for c in range(D)]
