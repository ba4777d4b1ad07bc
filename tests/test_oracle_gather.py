"""Pins for the oracle's dequantizing gather and for the byte order of a swapped
block record.

The gather is the fused read of "vLLM 0.7 Ships Unified KV Cache Compression",
"Technical Breakdown", step 4: an outlier channel takes its fp16 value from the
outlier buffer, every other channel is e2m1(code) x e4m3(group scale); an FP8
value is decode(code) x the block's K or V scale ("vLLM v0.7.2" field report,
"Deconstructing the v0.7.2 Architecture"), reached through the block table
("vLLM" glossary, "PagedAttention").

The expected values here are decoded from the raw cache bytes without the
oracle: FP8 and E4M3 codes through PyTorch's float8 dtypes, E2M1 codes through
the published code table (tests/golden/ocp_formats.json), fp16 outlier values
through NumPy's float16, and every byte position from the layout include/pqkv.h
states. The oracle's gather must equal that decoding bit for bit (both are one
fp64 product of two exactly decoded numbers), and stay within the quantizers'
error bounds of the values that were written.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import random_tables, slots, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ocp_formats.json")
FPMAX = {oracle.DT_E4M3: 448.0, oracle.DT_E5M2: 57344.0}
TORCH_FP8 = {oracle.DT_E4M3: torch.float8_e4m3fn, oracle.DT_E5M2: torch.float8_e5m2}


def _e2m1_table():
    with open(GOLDEN) as f:
        codes = json.load(f)["e2m1"]["codes"]
    t = np.zeros(16, dtype=np.float64)
    for k, v in codes.items():
        t[int(k, 16)] = v
    return t


E2M1 = _e2m1_table()


def _fp8_values(c, dt):
    """Every code of the cache as float64, shaped [nb][H][2][16][D] (header layout)."""
    codes = torch.from_numpy(c.cache.reshape(c.nb, c.H, 2, 16, c.D).copy())
    return codes.view(TORCH_FP8[dt]).to(torch.float64).numpy()


def numpy_gather_fp8(c, dt, table_row, L, h):
    vals = _fp8_values(c, dt)
    sc = c.scales.view(np.float32).reshape(c.nb, c.H, 4).astype(np.float64)  # {s_K, s_V, 0, 0}
    k = np.empty((L, c.D))
    v = np.empty((L, c.D))
    for t in range(L):
        blk, o = int(table_row[t // 16]), t % 16
        k[t] = vals[blk, h, 0, o] * sc[blk, h, 0]
        v[t] = vals[blk, h, 1, o] * sc[blk, h, 1]
    return k, v


def _v_pair_row(o):
    """Row of the FP4 V tile holding token offset o (channels [0, D/2)), and its nibble."""
    p = 2 * (o // 2) if o < 8 else 2 * ((o - 8) // 2) + 1
    return p, 4 * (o & 1)


def numpy_gather_fp4(c, table_row, L, h):
    nb, H, D = c.nb, c.H, c.D
    rows = c.cache.reshape(nb, H, 2, 16, D // 2)
    scl = torch.from_numpy(c.scales.reshape(nb, H, 2, 16, D // 16).copy()).view(torch.float8_e4m3fn)
    scl = scl.to(torch.float64).numpy()
    idx = c.oidx.reshape(nb, H, 2, 8)
    val = c.oval.view(np.float16).reshape(nb, H, 2, 16, 4).astype(np.float64)
    out = [np.empty((L, D)), np.empty((L, D))]
    for t in range(L):
        blk, o = int(table_row[t // 16]), t % 16
        kb = rows[blk, h, 0, o].astype(np.int64)
        kcodes = np.empty(D, dtype=np.int64)
        kcodes[0::2] = kb & 0xF
        kcodes[1::2] = kb >> 4
        p, shift = _v_pair_row(o)
        vb = np.concatenate([rows[blk, h, 1, p], rows[blk, h, 1, 8 + p]]).astype(np.int64)
        vcodes = (vb >> shift) & 0xF
        for kv, codes in ((0, kcodes), (1, vcodes)):
            x = E2M1[codes] * np.repeat(scl[blk, h, kv, o], 16)
            for r in range(4):
                ch = int(idx[blk, h, kv, r])
                if ch != 0xFF:
                    x[ch] = val[blk, h, kv, o, r]
            out[kv][t] = x
    return out[0], out[1]


def _fp8_spacing(dt, y):
    mbits, emin = (3, -6) if dt == oracle.DT_E4M3 else (2, -14)
    e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** emin)))
    return 2.0 ** (e - mbits)


def _data(rng, L, H, D, kv):
    """K and V of very different size, every head its own size, every token its
    own size: a K/V, head or token mix-up in the read changes the values."""
    head = np.array([1.0, 7.0, 0.2, 30.0][:H], dtype=np.float32)[None, :, None]
    tok = np.exp(rng.standard_normal((L, 1, 1))).astype(np.float32)
    base = 3.0 if kv == 0 else 0.01
    return rng.standard_normal((L, H, D), dtype=np.float32) * head * tok * base


@pytest.mark.parametrize("dt", [oracle.DT_E4M3, oracle.DT_E5M2])
@pytest.mark.parametrize("D", [64, 128])
def test_fp8_gather_equals_an_independent_decode_of_the_bytes(dt, D):
    rng = np.random.default_rng(31 + dt + D)
    H, nb = 3, 48
    lens = [37, 16, 70, 1]
    bt = random_tables(rng, lens, nb)
    c = oracle.Cache(dt, nb, H, D)
    written = []
    for b, L in enumerate(lens):
        k = torch.from_numpy(_data(rng, L, H, D, 0)).to(torch.bfloat16)
        v = torch.from_numpy(_data(rng, L, H, D, 1)).to(torch.bfloat16)
        written.append((to_f64(k), to_f64(v)))
        assert oracle.kv_cache_write(c, k, v, slots(bt[b], 0, L)) == 0
    sc = c.scales.view(np.float32).reshape(nb, H, 4)
    for b, L in enumerate(lens):
        for h in range(H):
            kd, vd, valid = oracle.gather(c, bt[b], L, h)
            assert valid.all()
            ke, ve = numpy_gather_fp8(c, dt, bt[b], L, h)
            np.testing.assert_array_equal(kd, ke)
            np.testing.assert_array_equal(vd, ve)
            for kv, got in ((0, kd), (1, vd)):
                x = written[b][kv][:, h]
                s = np.repeat(sc[bt[b][:(L + 15) // 16], h, kv].astype(np.float64), 16)[:L, None]
                bound = s * _fp8_spacing(dt, x / s) / 2 * (1 + 1e-6) + 1e-30
                assert (np.abs(got - x) <= bound).all()


def _fp4_data(rng, L, H, D):
    """N(0,1) with per-(head, K|V) planted x16 channels (different for K and V
    and for every head) and per-token sizes; returns x [2][L][H][D] and the
    planted channels [H][2][2]."""
    x = np.stack([_data(rng, L, H, D, 0), _data(rng, L, H, D, 1)])
    ch = np.empty((H, 2, 2), dtype=np.int64)
    for h in range(H):
        for kv in range(2):
            ch[h, kv] = np.sort(rng.choice(D, size=2, replace=False))
            x[kv, :, h, ch[h, kv]] *= 16.0
    return x, ch


@pytest.mark.parametrize("D", [64, 128])
def test_fp4_gather_equals_an_independent_decode_of_the_bytes(D):
    rng = np.random.default_rng(77 + D)
    H, nb = 3, 64
    lens = [64, 33, 16, 100]
    bt = random_tables(rng, lens, nb)
    c = oracle.Cache(oracle.DT_E2M1, nb, H, D)
    written = []
    for b, L in enumerate(lens):
        x, _ = _fp4_data(rng, L, H, D)
        k = torch.from_numpy(x[0]).to(torch.bfloat16)
        v = torch.from_numpy(x[1]).to(torch.bfloat16)
        written.append((to_f64(k), to_f64(v)))
        # block-aligned chunks of 32 tokens, so every block's outlier set comes
        # from its own 16 (or fewer, at the end) tokens
        for c0 in range(0, L, 32):
            c1 = min(L, c0 + 32)
            assert oracle.kv_cache_write(c, k[c0:c1].contiguous(), v[c0:c1].contiguous(),
                                         slots(bt[b], c0, c1 - c0)) == 0
    idx = c.oidx.reshape(nb, H, 2, 8)
    scl = torch.from_numpy(c.scales.reshape(nb, H, 2, 16, D // 16).copy()).view(torch.float8_e4m3fn)
    scl = scl.to(torch.float64).numpy()
    n_out = 0
    for b, L in enumerate(lens):
        for h in range(H):
            kd, vd, valid = oracle.gather(c, bt[b], L, h)
            assert valid.all()
            ke, ve = numpy_gather_fp4(c, bt[b], L, h)
            np.testing.assert_array_equal(kd, ke)
            np.testing.assert_array_equal(vd, ve)
            for kv, got in ((0, kd), (1, vd)):
                x = written[b][kv][:, h]
                for t in range(L):
                    blk, o = int(bt[b][t // 16]), t % 16
                    outs = [int(i) for i in idx[blk, h, kv, :4] if i != 0xFF]
                    n_out += len(outs)
                    # outlier channels: the fp16 of the written value
                    for ch in outs:
                        assert got[t, ch] == float(np.float16(x[t, ch]))
                    # the rest: within the E2M1 rounding of x / scale, or its clip at 6;
                    # a group scale that rounded to E4M3 zero (absmax / 6 at most half the
                    # smallest subnormal, 2^-10) reads as zero
                    rest = np.array([ch for ch in range(D) if ch not in outs])
                    sd = np.repeat(scl[blk, h, kv, o], 16)[rest]
                    xr, gr = x[t, rest], got[t, rest]
                    z = sd == 0
                    assert (gr[z] == 0).all() and (np.abs(xr[z]) <= 6 * 2.0 ** -10 * (1 + 1e-6)).all()
                    y = np.where(z, 0.0, xr / np.where(z, 1.0, sd))
                    spacing = np.where(np.abs(y) < 2, 0.5, np.where(np.abs(y) < 4, 1.0, 2.0))
                    bound = sd * np.maximum(spacing / 2, np.abs(y) - 6) * (1 + 1e-6) + 1e-30
                    assert (np.abs(gr[~z] - xr[~z]) <= bound[~z]).all()
    assert n_out > 0


def test_fp4_gather_of_hand_built_bytes():
    """One block written byte by byte from the header's layout (no write call):
    K token t channel c has code (t + c) % 16, V token t channel c code
    (3t + c) % 16; group scales 2^(t % 4 - 1) for K and 2^-(g % 3) for V;
    outlier slots K {5, 70}, V {0, 127} with values t + r / 4 (K) and -(t + r) (V)."""
    D, H = 128, 1
    c = oracle.Cache(oracle.DT_E2M1, 1, H, D)
    rows = c.cache.reshape(1, H, 2, 16, D // 2)
    t = np.arange(16)[:, None]
    ch = np.arange(D)[None, :]
    kc = (t + ch) % 16
    vc = (3 * t + ch) % 16
    rows[0, 0, 0] = (kc[:, 0::2] | (kc[:, 1::2] << 4)).astype(np.uint8)
    half = D // 2
    for o in range(16):
        p, shift = _v_pair_row(o)
        for part in range(2):
            r = rows[0, 0, 1, 8 * part + p]
            cur = r.astype(np.int64) & ~(0xF << shift) & 0xFF
            rows[0, 0, 1, 8 * part + p] = (cur | (vc[o, part * half:(part + 1) * half] << shift)).astype(np.uint8)
    e4m3 = {0.5: 0x30, 1.0: 0x38, 2.0: 0x40, 4.0: 0x48, 0.25: 0x28}  # OCP OFP8 E4M3 codes
    scl = c.scales.reshape(1, H, 2, 16, D // 16)
    ks = np.array([2.0 ** (o % 4 - 1) for o in range(16)])
    vs = np.array([2.0 ** -(g % 3) for g in range(D // 16)])
    for o in range(16):
        scl[0, 0, 0, o] = e4m3[ks[o]]
        scl[0, 0, 1, o] = [e4m3[s] for s in vs]
    idx = c.oidx.reshape(1, H, 2, 8)
    idx[0, 0, 0] = [5, 70, 0xFF, 0xFF, 0xFF, 0xFF, 0xFF, 0xFF]
    idx[0, 0, 1] = [0, 127, 0xFF, 0xFF, 0xFF, 0xFF, 0xFF, 0xFF]
    val = c.oval.view(np.float16).reshape(1, H, 2, 16, 4)
    val[0, 0, 0] = np.array([[o + r / 4 for r in range(4)] for o in range(16)], dtype=np.float16)
    val[0, 0, 1] = np.array([[-(o + r) for r in range(4)] for o in range(16)], dtype=np.float16)
    kd, vd, valid = oracle.gather(c, np.array([0], np.int32), 16, 0)
    assert valid.all()
    kw = E2M1[kc] * ks[:, None]
    kw[:, 5] = np.arange(16)
    kw[:, 70] = np.arange(16) + 0.25
    vw = E2M1[vc] * np.repeat(vs, 16)[None, :]
    vw[:, 0] = -np.arange(16)
    vw[:, 127] = -(np.arange(16) + 1)
    np.testing.assert_array_equal(kd, kw)
    np.testing.assert_array_equal(vd, vw)


def test_fp8_gather_of_hand_built_bytes():
    """One E4M3 block set byte by byte: code of token t channel c = (t * 8 + c) % 126
    (all finite), K scale 0.5, V scale 3.0."""
    D, H = 64, 2
    c = oracle.Cache(oracle.DT_E4M3, 2, H, D)
    codes = c.cache.reshape(2, H, 2, 16, D)
    t = np.arange(16)[:, None]
    chn = np.arange(D)[None, :]
    code = ((t * 8 + chn) % 126).astype(np.uint8)
    codes[1, 1, 0] = code
    codes[1, 1, 1] = code ^ 0x80  # negated
    c.scales.view(np.float32).reshape(2, H, 4)[1, 1] = [0.5, 3.0, 0.0, 0.0]
    kd, vd, valid = oracle.gather(c, np.array([1], np.int32), 16, 1)
    dec = torch.from_numpy(code.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(kd, dec * 0.5)
    np.testing.assert_array_equal(vd, -dec * 3.0)


@pytest.mark.parametrize("dt", [oracle.DT_BF16, oracle.DT_E4M3, oracle.DT_E2M1])
def test_swap_record_is_the_header_byte_order(dt):
    """include/pqkv.h: a record is the block's cache bytes (all heads, K and V),
    then its scales, outlier indices and outlier values, each in the cache's own
    layout. Each array of a block gets its own marker byte pattern; the record
    must hold the patterns in that order and nothing else."""
    H, D, nb = 2, 64, 5
    c = oracle.Cache(dt, nb, H, D, poison=False)
    shapes = {oracle.DT_BF16: [(H, 2, 16, D * 2)],
              oracle.DT_E4M3: [(H, 2, 16, D), (H, 4 * 4)],
              oracle.DT_E2M1: [(H, 2, 16, D // 2), (H, 2, 16, D // 16), (H, 2, 8), (H, 2, 16, 4 * 2)]}[dt]
    arrays = [a for a in c.arrays() if a is not None]
    assert len(arrays) == len(shapes)
    expect = []
    for i, (a, shp) in enumerate(zip(arrays, shapes)):
        per_block = int(np.prod(shp))
        assert a.size == nb * per_block
        blocks = a.reshape(nb, per_block)
        for b in range(nb):
            blocks[b] = (np.arange(per_block) * 7 + 16 * i + 64 * b) % 251
        expect.append(blocks[3].copy())
    rec_bytes = sum(int(np.prod(s)) for s in shapes)
    assert oracle.block_record_bytes(dt, H, D) == rec_bytes
    rec = np.zeros((2, rec_bytes), dtype=np.uint8)
    assert oracle.swap_out(c, [3, 1], rec) == 0
    np.testing.assert_array_equal(rec[0], np.concatenate(expect))
    off = 0
    for i, (a, shp) in enumerate(zip(arrays, shapes)):
        n = int(np.prod(shp))
        np.testing.assert_array_equal(rec[1, off:off + n], a.reshape(nb, n)[1])
        off += n
