"""Pins for the oracle's quantizing cache write.

Checked against: hand-worked examples (tests/golden/hand_write_examples.json),
exact round trips for the 16-bit formats, the quantizers' own error bounds and
scale statistics, NumPy's population mean/std and float16 cast (library
routines) for the outlier selection and the FP16 outlier buffer, and the
closed form of equal channel norms (zero variance).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import random_tables, slots, to_f64

HAND = os.path.join(os.path.dirname(__file__), "golden", "hand_write_examples.json")
FPMAX = {oracle.DT_E4M3: 448.0, oracle.DT_E5M2: 57344.0}


def _hand():
    with open(HAND) as f:
        return json.load(f)


def _row(spec, D):
    rest = spec.get("_rest", 0.0)
    r = np.full(D, rest, dtype=np.float32)
    for k, v in spec.items():
        if k != "_rest":
            r[int(k)] = v
    return r


def _codes(spec, D):
    rest = int(spec.get("_rest", "0x00"), 16)
    r = np.full(D, rest, dtype=np.uint8)
    for k, v in spec.items():
        if k != "_rest":
            r[int(k)] = int(v, 16)
    return r


def _fp8_view(c):
    nb, H, D = c.nb, c.H, c.D
    return c.cache.reshape(nb, H, 2, 16, D), c.scales.view(np.float32).reshape(nb, H, 4)


def test_fp8_hand_example():
    g = _hand()["fp8_e4m3"]
    D, H, nb = g["head_dim"], g["num_kv_heads"], g["num_blocks"]
    c = oracle.Cache(oracle.DT_E4M3, nb, H, D)

    def tok(spec):
        return torch.from_numpy(_row(spec, D)[None, None, :]).to(torch.bfloat16)

    assert oracle.kv_cache_write(c, tok(g["k_token0"]), tok(g["v_token0"]), np.array([0], np.int32)) == 0
    codes, sc = _fp8_view(c)
    a = g["after_call1"]
    assert sc[0, 0, 0] == a["scale_k"] and sc[0, 0, 1] == a["scale_v"]
    np.testing.assert_array_equal(codes[0, 0, 0, 0], _codes(a["k_codes_offset0"], D))
    np.testing.assert_array_equal(codes[0, 0, 1, 0], _codes(a["v_codes_offset0"], D))
    assert (codes[0, 0, :, 1:] == 0xFF).all()  # untouched slots keep the poison
    assert oracle.kv_cache_write(c, tok(g["k_token1"]), tok(g["v_token1"]), np.array([1], np.int32)) == 0
    a = g["after_call2"]
    assert sc[0, 0, 0] == a["scale_k"] and sc[0, 0, 1] == a["scale_v"]
    np.testing.assert_array_equal(codes[0, 0, 0, 0], _codes(a["k_codes_offset0"], D))
    np.testing.assert_array_equal(codes[0, 0, 0, 1], _codes(a["k_codes_offset1"], D))
    np.testing.assert_array_equal(codes[0, 0, 1, 0], _codes(a["v_codes_offset0"], D))
    np.testing.assert_array_equal(codes[0, 0, 1, 1], _codes(a["v_codes_offset1"], D))


def test_fp4_hand_example():
    g = _hand()["fp4"]
    D, H, nb = g["head_dim"], g["num_kv_heads"], g["num_blocks"]
    sign = np.where(np.arange(D) % 2 == 0, 1.0, -1.0).astype(np.float32)
    k = np.tile(sign, (16, H, 1))
    k[:, :, 5] = 100.0
    k[:, :, 40] = -50.0
    v = np.tile(sign, (16, H, 1))
    c = oracle.Cache(oracle.DT_E2M1, nb, H, D)
    kt = torch.from_numpy(k).to(torch.bfloat16)
    vt = torch.from_numpy(v).to(torch.bfloat16)
    assert oracle.kv_cache_write(c, kt, vt, np.arange(16, dtype=np.int32)) == 0
    rows = c.cache.reshape(nb, H, 2, 16, D // 2)
    scl = c.scales.reshape(nb, H, 2, 16, D // 16)
    idx = c.oidx.reshape(nb, H, 2, 8)
    val = c.oval.view(np.uint16).reshape(nb, H, 2, 16, 4)
    hexs = lambda xs: np.array([int(x, 16) for x in xs])
    for t in range(16):
        np.testing.assert_array_equal(rows[0, 0, 0, t], hexs(g["k_row_bytes"]))
        want_v = g["v_rows_0_to_7"] if t < 8 else g["v_rows_8_to_15"]
        np.testing.assert_array_equal(rows[0, 0, 1, t], hexs(want_v))
    for kv, name in ((0, "k"), (1, "v")):
        for t in range(16):
            np.testing.assert_array_equal(scl[0, 0, kv, t], hexs(g[name + "_scales"]))
            np.testing.assert_array_equal(val[0, 0, kv, t], hexs(g[name + "_vals"]))
        np.testing.assert_array_equal(idx[0, 0, kv], hexs(g[name + "_idx"]))
    assert (rows[1] == 0xFF).all()


# E2M1 magnitudes in code order (OCP Microscaling Formats, E2M1).
_E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


@pytest.mark.parametrize("D", [64, 128])
def test_fp4_v_tile_pair_order(D):
    """The V tile's storage order as include/pqkv.h states it: one byte holds one
    channel of a token pair, pair p = 2k is tokens (2k, 2k+1), pair 2k+1 is tokens
    (2k+8, 2k+9), even token in the low nibble, channels [0, D/2) in row p and
    [D/2, D) in row 8+p. Each token gets codes known by construction: channel c of
    token t is the E2M1 value of magnitude code (t + 3c) % 8 with sign (-1)^(c // 2)
    (zero kept positive),
    so every 16-channel group reaches 6 (scale 6/6 = 1, exact) and every channel
    reaches norm 6 (variance 0: channels 0-3 are the outliers, their codes 0)."""
    t = np.arange(16)[:, None]
    c = np.arange(D)[None, :]
    mag = (t + 3 * c) % 8
    sign = np.where((c // 2) % 2 == 0, 1.0, -1.0)
    x = np.where(mag == 0, 0.0, np.array(_E2M1_MAGS)[mag] * sign).astype(np.float32)[:, None, :]
    code = mag | np.where((sign < 0) & (mag > 0), 8, 0)
    code[:, :4] = 0
    cache = oracle.Cache(oracle.DT_E2M1, 1, 1, D)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    assert oracle.kv_cache_write(cache, xt, xt, np.arange(16, dtype=np.int32)) == 0
    rows, scl, idx, _ = _fp4_views(cache)
    assert list(idx[0, 0, 1][:4]) == [0, 1, 2, 3]
    assert (scl[0, 0, 1] == 0x38).all()  # E4M3 1.0
    half = D // 2
    for p in range(8):
        ta = p if p % 2 == 0 else p + 7
        for part in range(2):
            chans = np.arange(half) + part * half
            want = code[ta, chans] | (code[ta + 1, chans] << 4)
            np.testing.assert_array_equal(rows[0, 0, 1, 8 * part + p], want)
    # K keeps one row per token, channel 2i in the low nibble
    np.testing.assert_array_equal(_fp4_codes(rows[0, 0, 0]), code)


@pytest.mark.parametrize("dt", [oracle.DT_FP16, oracle.DT_BF16])
def test_16bit_write_is_exact_and_touches_only_its_slots(dt):
    rng = np.random.default_rng(1)
    H, D, nb = 3, 64, 20
    lens = [5, 16, 33]
    bt = random_tables(rng, lens, nb)
    c = oracle.Cache(dt, nb, H, D)
    ind = torch.float16 if dt == oracle.DT_FP16 else torch.bfloat16
    kvs = []
    for b, L in enumerate(lens):
        k = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(ind)
        v = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(ind)
        kvs.append((k, v))
        oracle.kv_cache_write(c, k, v, slots(bt[b], 0, L))
    for b, L in enumerate(lens):
        for h in range(H):
            kd, vd, _ = oracle.gather(c, bt[b], L, h)
            np.testing.assert_array_equal(kd, to_f64(kvs[b][0][:, h]))
            np.testing.assert_array_equal(vd, to_f64(kvs[b][1][:, h]))
    written = sum(lens) * H * 2 * D * 2
    assert (c.cache != 0xFF).sum() <= written
    assert (c.cache == 0xFF).sum() >= c.cache.size - written


def _fp8_spacing(dt, y):
    """Distance between neighbouring codes around |y| (format units)."""
    mbits, emin = (3, -6) if dt == oracle.DT_E4M3 else (2, -14)
    e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** emin)))
    return 2.0 ** (e - mbits)


@pytest.mark.parametrize("dt", [oracle.DT_E4M3, oracle.DT_E5M2])
def test_fp8_scale_statistics_and_error_bound(dt):
    rng = np.random.default_rng(2 + dt)
    H, D, nb = 2, 64, 32
    lens = [16, 40, 7]
    bt = random_tables(rng, lens, nb)
    c = oracle.Cache(dt, nb, H, D)
    data = []
    for b, L in enumerate(lens):
        k = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32) * 3).to(torch.bfloat16)
        v = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32) * 0.01).to(torch.bfloat16)
        data.append((k, v))
        oracle.kv_cache_write(c, k, v, slots(bt[b], 0, L))
    codes, sc = _fp8_view(c)
    for b, L in enumerate(lens):
        for j in range((L + 15) // 16):
            blk = bt[b, j]
            n = min(16, L - 16 * j)
            for h in range(H):
                for kv in range(2):
                    x = to_f64(data[b][kv][16 * j:16 * j + n, h])
                    s = float(sc[blk, h, kv])
                    assert s == np.float32(np.float32(np.abs(x).max()) / np.float32(FPMAX[dt]))
                    dec = oracle.decode(dt, codes[blk, h, kv, :n].ravel()).reshape(n, D)
                    assert np.abs(dec).max() == FPMAX[dt]
                    err = np.abs(dec * s - x)
                    bound = s * _fp8_spacing(dt, x / s) / 2 * (1 + 1e-6) + 1e-30
                    assert (err <= bound).all()


@pytest.mark.parametrize("dt", [oracle.DT_E4M3, oracle.DT_E5M2])
def test_fp8_append_grows_scale_and_reencodes(dt):
    rng = np.random.default_rng(5 + dt)
    H, D, nb = 1, 64, 4
    c = oracle.Cache(dt, nb, H, D)
    k1 = torch.from_numpy(rng.standard_normal((5, H, D), dtype=np.float32)).to(torch.bfloat16)
    oracle.kv_cache_write(c, k1, k1, np.arange(5, dtype=np.int32) + 16)
    codes, sc = _fp8_view(c)
    before = codes[1, 0, 0, :5].copy()
    s_old = float(sc[1, 0, 0])
    # smaller values: scale and old codes unchanged
    k2 = (k1[:2].float() * 0.25).to(torch.bfloat16)
    oracle.kv_cache_write(c, k2, k2, np.arange(5, 7, dtype=np.int32) + 16)
    assert float(sc[1, 0, 0]) == s_old
    np.testing.assert_array_equal(codes[1, 0, 0, :5], before)
    # larger values: scale = new absmax / FPMAX, old codes re-encoded
    k3 = (k1[:3].float() * 8).to(torch.bfloat16)
    oracle.kv_cache_write(c, k3, k3, np.arange(7, 10, dtype=np.int32) + 16)
    s_new = float(sc[1, 0, 0])
    assert s_new == np.float32(np.float32(np.abs(to_f64(k3)).max()) / np.float32(FPMAX[dt]))
    old_vals = oracle.decode(dt, before.ravel()) * s_old
    new_vals = oracle.decode(dt, codes[1, 0, 0, :5].ravel()) * s_new
    bound = s_new * _fp8_spacing(dt, old_vals / s_new) / 2 * (1 + 1e-6) + 1e-30
    assert (np.abs(new_vals - old_vals) <= bound).all()


def test_fp8_zero_block_has_zero_scale_and_codes():
    c = oracle.Cache(oracle.DT_E4M3, 2, 1, 64)
    z = torch.zeros((3, 1, 64), dtype=torch.bfloat16)
    oracle.kv_cache_write(c, z, z, np.arange(3, dtype=np.int32))
    codes, sc = _fp8_view(c)
    assert sc[0, 0, 0] == 0 and sc[0, 0, 1] == 0 and (codes[0, 0, :, :3] == 0).all()


def _fp4_views(c):
    nb, H, D = c.nb, c.H, c.D
    return (c.cache.reshape(nb, H, 2, 16, D // 2), c.scales.reshape(nb, H, 2, 16, D // 16),
            c.oidx.reshape(nb, H, 2, 8), c.oval.view(np.uint16).reshape(nb, H, 2, 16, 4))


def _fp4_codes(rows):
    lo = rows & 0xF
    hi = rows >> 4
    return np.stack([lo, hi], axis=-1).reshape(rows.shape[:-1] + (rows.shape[-1] * 2,))


def _numpy_outliers(x):
    """Library-routine restatement: numpy mean/std (population) of the channel norms."""
    n = np.abs(x).max(axis=0)
    thr = n.mean() + 3.2 * n.std()
    cand = [c for c in range(len(n)) if n[c] >= thr]
    cand.sort(key=lambda c: (-n[c], c))
    return sorted(cand[:4]), n, thr


def test_fp4_outlier_selection_matches_numpy_statistics():
    rng = np.random.default_rng(7)
    H, D, nb = 4, 128, 64
    c = oracle.Cache(oracle.DT_E2M1, nb, H, D)
    checked = 0
    for blk in range(nb):
        # heavy-tailed channels give anywhere from 0 to many flagged channels
        gains = np.exp(rng.standard_normal((H, D)) * rng.uniform(0.1, 1.5))
        x = rng.standard_normal((16, H, D)).astype(np.float32) * gains[None].astype(np.float32)
        t = torch.from_numpy(x).to(torch.bfloat16)
        oracle.kv_cache_write(c, t, t, np.arange(16, dtype=np.int32) + 16 * blk)
        _, _, idx, val = _fp4_views(c)
        xf = to_f64(t)
        for h in range(H):
            want, n, thr = _numpy_outliers(xf[:, h])
            if np.min(np.abs(n - thr)) < 1e-9 * thr:
                continue
            got = [int(i) for i in idx[blk, h, 0] if i != 0xFF]
            assert got == want
            with np.errstate(over="ignore"):
                ref_vals = xf[:, h][:, want].astype(np.float32).astype(np.float16).view(np.uint16)
            np.testing.assert_array_equal(val[blk, h, 0][:, :len(want)], ref_vals)
            assert (val[blk, h, 0][:, len(want):] == 0).all()
            checked += 1
    assert checked > 200


def test_fp4_equal_norms_flag_the_lowest_channels():
    D = 64
    x = np.ones((16, 1, D), dtype=np.float32)
    x[:, :, 1::2] = -1
    t = torch.from_numpy(x).to(torch.bfloat16)
    c = oracle.Cache(oracle.DT_E2M1, 1, 1, D)
    oracle.kv_cache_write(c, t, t, np.arange(16, dtype=np.int32))
    _, _, idx, _ = _fp4_views(c)
    assert list(idx[0, 0, 0]) == [0, 1, 2, 3, 255, 255, 255, 255]


def test_fp4_planted_outlier_channels_are_found():
    import workloads
    s = workloads.spec("fp4", batch=2)
    tab = workloads.tables(s)
    ch = workloads.outlier_channels(s)
    c = oracle.Cache(oracle.DT_E2M1, int(tab.block_tables.max()) + 1, s.num_kv_heads, s.head_dim)
    full = hits = 0
    for b in range(2):
        k, v = workloads.seq_kv(s, b)
        L = k.shape[0]
        n = min(L, 2048)
        oracle.kv_cache_write(c, k[:n], v[:n], workloads.slots_for(tab.block_tables[b], 0, n))
        _, _, idx, _ = _fp4_views(c)
        for j in range(n // 16):
            blk = tab.block_tables[b, j]
            for h in range(s.num_kv_heads):
                for kv in range(2):
                    got = [int(i) for i in idx[blk, h, kv] if i != 0xFF]
                    full += 1
                    hits += got == list(ch[h, kv])
    assert hits >= 0.99 * full


def test_fp4_group_bound_and_error_bound():
    rng = np.random.default_rng(9)
    H, D, nb = 2, 128, 8
    c = oracle.Cache(oracle.DT_E2M1, nb, H, D)
    x = (rng.standard_normal((40, H, D)) * np.exp(rng.standard_normal((1, H, D)))).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16)
    oracle.kv_cache_write(c, t[:16], t[:16], np.arange(16, dtype=np.int32))
    oracle.kv_cache_write(c, t[16:20], t[16:20], np.arange(32, 36, dtype=np.int32))
    idx_after_first = c.oidx.reshape(nb, H, 2, 8)[2].copy()
    # a later run in block 2 (offsets 4..15) reuses the outlier set of its first write
    oracle.kv_cache_write(c, t[20:40], t[20:40], np.arange(36, 56, dtype=np.int32))
    np.testing.assert_array_equal(c.oidx.reshape(nb, H, 2, 8)[2], idx_after_first)
    rows, scl, idx, _ = _fp4_views(c)
    xf = to_f64(t)
    tok_slots = list(range(0, 16)) + list(range(32, 56))
    for i, sl in enumerate(tok_slots):
        blk, off = sl // 16, sl % 16
        for h in range(H):
            codes = _fp4_codes(rows[blk, h, 0, off])
            e2 = oracle.decode(oracle.DT_E2M1, codes.astype(np.uint8))
            sd = oracle.decode(oracle.DT_E4M3, scl[blk, h, 0, off])
            outs = set(int(j) for j in idx[blk, h, 0] if j != 0xFF)
            assert np.abs(e2).max() <= 6
            for g in range(D // 16):
                chans = [ch for ch in range(16 * g, 16 * g + 16) if ch not in outs]
                for ch in chans:
                    y = xf[i, h, ch] / sd[g] if sd[g] else 0.0
                    spacing = 0.5 if abs(y) < 2 else (1.0 if abs(y) < 4 else 2.0)
                    err = abs(e2[ch] * sd[g] - xf[i, h, ch])
                    bound = sd[g] * max(spacing / 2, abs(y) - 6) * (1 + 1e-6) + 1e-30
                    assert err <= bound
                for ch in outs:
                    assert codes[ch] == 0


def test_write_error_bits():
    c = oracle.Cache(oracle.DT_E4M3, 2, 1, 64)
    x = torch.ones((3, 1, 64), dtype=torch.bfloat16)
    assert oracle.kv_cache_write(c, x, x, np.array([0, 40, -1], np.int32)) == oracle.ERR_SLOT
    assert oracle.kv_cache_write(c, x, x, np.array([3, 5, 6], np.int32)) == oracle.ERR_RUN
    assert oracle.kv_cache_write(c, x, x, np.array([17, 18, 19], np.int32)) == 0


def test_bytes_per_token_against_the_pages_ratio():
    # 'vLLM 0.7 Ships Unified KV Cache Compression': 1.2 MB -> 0.34 MB per token
    # (a 72% reduction); the FP4 codes with one 8-bit scale per 16 channels give
    # 4.5 bits per element, 1152 of 4096 bytes per token (8 KV heads, D 128).
    H, D = 8, 128
    per_tok = lambda dt: sum(oracle.cache_sizes(dt, 1, H, D)) / 16
    bf16 = per_tok(oracle.DT_BF16)
    fp4_codes_scales = (oracle.cache_sizes(oracle.DT_E2M1, 1, H, D)[0] +
                        oracle.cache_sizes(oracle.DT_E2M1, 1, H, D)[1]) / 16
    assert bf16 == 4096 and fp4_codes_scales == 1152
    assert abs(fp4_codes_scales / bf16 - 0.34 / 1.2) < 0.005
    assert per_tok(oracle.DT_E4M3) == 2048 + 8  # one 16-byte scale granule per (block, head)
    assert per_tok(oracle.DT_E2M1) == 1024 + 128 + 8 + 128
