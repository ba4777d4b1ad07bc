"""Invariants of the decode's split of the KV work (host-side check of the design).

The decode lays the blocks of all (sequence, KV head) pairs end to end (T
blocks), gives warp w of W the blocks [w*Qw, (w+1)*Qw) with Qw = ceil(T/W), and,
with a fixed split of C blocks ("split-K over 512-token chunks": C = 32), also
cuts at every multiple of C. The cells between consecutive cuts are units,
counted in O(1) as unit(f) = f//C + f//Qw - f//lcm(C, Qw) (this restates the
kernel's formula). A pair's pieces are the units its blocks cross; a piece that
continues an earlier piece writes slot 2k of its unit k, a piece that starts in
unit k and continues after it writes slot 2k + 1, and a pair inside one unit
writes no slot. The workspace holds 2 slots per chunk, chunks =
ceil(B * Hkv * max_blocks / C) + W (or W for the balanced split).

These tests check, over random plans, what the kernel relies on: units advance by
one exactly at the cuts, a pair's pieces are consecutive units, no two pieces
share a slot, and every slot lies inside the workspace.
"""
import math

import numpy as np
import pytest


def unit(f, C, Qw, lcm):
    return f // C + f // Qw - f // lcm


def plan(T, W, C):
    Qw = max(1, -(-T // W))
    C = C if C > 0 else Qw
    return Qw, C, Qw // math.gcd(Qw, C) * C


@pytest.mark.parametrize("seed", range(6))
def test_units_pieces_and_slots(seed):
    rng = np.random.default_rng(seed)
    for _ in range(500):
        B = int(rng.integers(1, 40))
        Hkv = int(rng.choice([1, 2, 8]))
        lens = rng.integers(0, 5000, size=B)
        nblk = (lens + 15) // 16
        maxblk = int(max(1, nblk.max()))
        W = int(rng.choice([148 * 5, 148 * 12, 148 * 8, 37]))
        split = int(rng.choice([0, 1, 3, 32, 1000]))
        T = int(Hkv * nblk.sum())
        if T == 0:
            continue
        Qw, C, lcm = plan(T, W, split)
        # units advance by one exactly where a block starts at a cut
        f = np.arange(T)
        u = unit(f, C, Qw, lcm)
        cut = (f % C == 0) | (f % Qw == 0)
        assert u[0] == 0
        assert np.array_equal(np.diff(u), cut[1:].astype(np.int64))
        chunks = (-(-B * Hkv * maxblk // split) + W) if split > 0 else W
        used = set()
        start = 0
        for b in range(B):
            for h in range(Hkv):
                n = int(nblk[b])
                if n == 0:
                    continue
                s0, s1 = start, start + n - 1
                start += n
                k0, k1 = int(u[s0]), int(u[s1])
                # the pair's pieces are the consecutive units k0..k1
                assert set(u[s0:s1 + 1].tolist()) == set(range(k0, k1 + 1))
                if k0 == k1:
                    continue  # whole inside one unit: written straight to the output
                for k in range(k0, k1 + 1):
                    slot = 2 * k if k > k0 else 2 * k + 1
                    assert slot not in used, "two pieces share slot %d" % slot
                    used.add(slot)
                    assert slot < 2 * chunks, "slot beyond the workspace"
        assert start == T


def test_512_token_split_of_the_llama70b_layer():
    """The Llama-3.1-70B-shaped layer (16 sequences of 24-40k tokens, 8 KV heads)
    at C = 32 blocks: every piece lies inside one 512-token chunk, and a pair of
    2048+ blocks has at least 64 pieces."""
    rng = np.random.default_rng(7)
    lens = rng.integers(24576, 40961, size=16)
    nblk = (lens + 15) // 16
    T = int(8 * nblk.sum())
    for W in (148 * 5, 148 * 12):
        Qw, C, lcm = plan(T, W, 32)
        f = np.arange(T)
        u = unit(f, C, Qw, lcm)
        # a unit never spans a multiple of C
        first = np.r_[0, np.flatnonzero(np.diff(u)) + 1]
        last = np.r_[first[1:] - 1, T - 1]
        assert np.all(first // 32 == last // 32)
        start = 0
        for b in range(16):
            n = int(nblk[b])
            for _ in range(8):
                assert u[start + n - 1] - u[start] + 1 >= n // 32
                start += n
