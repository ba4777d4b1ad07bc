"""GPU encoders (the hardware cvt used by the cache write) against the oracle's
encoders, bit for bit: every float32 in the formats' working range, plus
random bit patterns over the whole float32 line."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")

FMTS = [(pq.FP8_E4M3, oracle.DT_E4M3), (pq.FP8_E5M2, oracle.DT_E5M2), (pq.FP4_E2M1, oracle.DT_E2M1)]


def _check(x: np.ndarray, code, odt):
    xg = torch.from_numpy(x).cuda()
    out = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    pq.encode(xg, code, out)
    got = out.cpu().numpy()
    want = oracle.encode(odt, x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(x[i]), hex(x.view(np.uint32)[i]), int(got[i]), int(want[i])) for i in bad[:8]]


@pytest.mark.parametrize("code,odt", FMTS, ids=["e4m3", "e5m2", "e2m1"])
def test_every_float_of_the_working_range(code, odt):
    # all float32 (both signs) with exponents from below half the smallest
    # subnormal quantum to beyond saturation, in chunks of 2^24 values
    lo_e = {pq.FP8_E4M3: -12, pq.FP8_E5M2: -19, pq.FP4_E2M1: -4}[code]
    hi_e = {pq.FP8_E4M3: 10, pq.FP8_E5M2: 17, pq.FP4_E2M1: 4}[code]
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in range(lo_e, hi_e + 1):
        bits = ((e + 127) << 23) | mant
        x = np.concatenate([bits, bits | 0x80000000]).view(np.float32)
        _check(x, code, odt)


@pytest.mark.parametrize("code,odt", FMTS, ids=["e4m3", "e5m2", "e2m1"])
def test_random_bit_patterns_and_specials(code, odt):
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 1 << 32, size=1 << 24, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-38, 3e38, -3e38, 1.0, -1.0], np.float32)
    _check(np.concatenate([x, specials]).astype(np.float32), code, odt)


@pytest.mark.slow
@pytest.mark.parametrize("code,odt", FMTS, ids=["e4m3", "e5m2", "e2m1"])
def test_all_two_to_the_32_inputs(code, odt):
    """Every float32 bit pattern except NaNs (outside the encoders' domain),
    in chunks of 2^26: GPU and oracle codes equal bit for bit."""
    chunk = 1 << 26
    for c0 in range(0, 1 << 32, chunk):
        bits = np.arange(c0, c0 + chunk, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        x = x[~np.isnan(x)]
        _check(x, code, odt)
