"""Pins for the oracle's number-format encoders and decoders.

The oracle's E4M3 / E5M2 / E2M1 / binary16 routines are checked against things
other than themselves: the published code tables (tests/golden/ocp_formats.json),
PyTorch's float8 and NumPy's float16 conversions (library routines), and an
independent nearest-value search written here from the definition of
round-to-nearest-even over the decoded value table.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ocp_formats.json")
FMT = {"e4m3": oracle.DT_E4M3, "e5m2": oracle.DT_E5M2, "e2m1": oracle.DT_E2M1}
NCODES = {"e4m3": 256, "e5m2": 256, "e2m1": 16}
MAXV = {"e4m3": 448.0, "e5m2": 57344.0, "e2m1": 6.0}
SIGN = {"e4m3": 0x80, "e5m2": 0x80, "e2m1": 0x8}


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("name", ["e4m3", "e5m2", "e2m1"])
def test_decode_matches_published_tables(name):
    g = _golden()[name]
    codes = np.array([int(c, 16) for c in g["codes"]], dtype=np.uint8)
    vals = oracle.decode(FMT[name], codes)
    for c, want, got in zip(g["codes"], g["codes"].values(), vals):
        assert got == want and np.signbit(got) == np.signbit(want), (name, c, got, want)
    for c in g.get("nan_codes", []):
        assert np.isnan(oracle.decode(FMT[name], np.array([int(c, 16)], np.uint8))[0])
    for c, s in g.get("inf_codes", {}).items():
        assert oracle.decode(FMT[name], np.array([int(c, 16)], np.uint8))[0] == float(s)


@pytest.mark.parametrize("name,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_decode_all_codes_matches_torch(name, tdt):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode(FMT[name], codes)
    ref = torch.from_numpy(codes).view(tdt).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert (ours[~nan] == ref[~nan]).all()
    assert (np.signbit(ours[~nan]) == np.signbit(ref[~nan])).all()


def _finite_codes(name):
    codes = np.arange(NCODES[name], dtype=np.uint8)
    vals = oracle.decode(FMT[name], codes)
    keep = np.isfinite(vals)
    return codes[keep], vals[keep]


@pytest.mark.parametrize("name", ["e4m3", "e5m2", "e2m1"])
def test_roundtrip_every_finite_code(name):
    codes, vals = _finite_codes(name)
    back = oracle.encode(FMT[name], vals.astype(np.float32))
    assert (back == codes).all()  # +0 and -0 stay distinct


def _nearest_even_reference(name, x):
    """Independent encoder: nearest value of the positive code table, ties to
    the code with an even last bit, saturating at the largest finite value."""
    codes, vals = _finite_codes(name)
    pos = vals >= 0
    pcodes = codes[pos & ~np.signbit(vals)]
    pvals = vals[pos & ~np.signbit(vals)]
    order = np.argsort(pvals)
    pcodes, pvals = pcodes[order], pvals[order]
    a = np.abs(x.astype(np.float64))
    a = np.minimum(a, pvals[-1])
    hi = np.clip(np.searchsorted(pvals, a, side="left"), 0, len(pvals) - 1)
    lo = np.clip(hi - 1, 0, len(pvals) - 1)
    dlo = a - pvals[lo]
    dhi = pvals[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((pcodes[hi] & 1) == 0))
    c = np.where(pick_hi, pcodes[hi], pcodes[lo]).astype(np.uint8)
    c = np.where(a == pvals[hi], pcodes[hi], c).astype(np.uint8)
    return np.where(np.signbit(x), c | SIGN[name], c).astype(np.uint8)


def _sweep_inputs(name, n_random=400000, seed=0):
    _, vals = _finite_codes(name)
    pv = np.unique(np.abs(vals))
    mids = (pv[1:] + pv[:-1]) / 2.0
    base = np.concatenate([pv, mids, [MAXV[name] * 1.5, MAXV[name] * 1e3, 1e30, 1e-30, 1e-45]])
    f = base.astype(np.float32)
    near = [f]
    for k in (1, 2, 3):
        near.append(np.nextafter(f, np.float32(np.inf)))
        near.append(np.nextafter(f, np.float32(0)))
        f = near[-2]
    rng = np.random.default_rng(seed)
    lo, hi = np.log2(pv[1]) - 4, np.log2(MAXV[name]) + 2
    rnd = (2.0 ** rng.uniform(lo, hi, n_random)).astype(np.float32)
    bits = rng.integers(0, 2 ** 32, size=n_random, dtype=np.uint64).astype(np.uint32).view(np.float32)
    bits = bits[np.isfinite(bits)]
    x = np.concatenate(near + [rnd, bits])
    return np.concatenate([x, -x]).astype(np.float32)


@pytest.mark.parametrize("name", ["e4m3", "e5m2", "e2m1"])
def test_encoder_equals_independent_nearest_even_search(name):
    x = _sweep_inputs(name)
    ours = oracle.encode(FMT[name], x)
    ref = _nearest_even_reference(name, x)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]


@pytest.mark.parametrize("name", ["e4m3", "e5m2", "e2m1"])
def test_ties_go_to_even_and_saturation(name):
    codes, vals = _finite_codes(name)
    pos = np.sort(np.unique(vals[vals > 0]))
    # exact midpoints between neighbours go to the even code
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32((a + b) / 2)
        if float(m) != (a + b) / 2:
            continue
        c = int(oracle.encode(FMT[name], np.array([m]))[0])
        assert c & 1 == 0, (name, a, b, c)
        up = np.nextafter(m, np.float32(np.inf))
        assert oracle.decode(FMT[name], oracle.encode(FMT[name], np.array([up])))[0] == b
    big = np.array([MAXV[name] * 1.01, MAXV[name] * 1e6, np.inf], np.float32)
    assert (oracle.decode(FMT[name], oracle.encode(FMT[name], big)) == MAXV[name]).all()
    assert (oracle.decode(FMT[name], oracle.encode(FMT[name], -big)) == -MAXV[name]).all()
    z = oracle.encode(FMT[name], np.array([0.0, -0.0, -1e-30], np.float32))
    assert list(z) == [0, SIGN[name], SIGN[name]]


@pytest.mark.parametrize("name,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_encoder_matches_torch_cast_in_range(name, tdt):
    x = _sweep_inputs(name, n_random=200000, seed=1)
    x = x[np.abs(x) <= MAXV[name]]
    ours = oracle.encode(FMT[name], x)
    ref = torch.from_numpy(x).to(tdt).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]


def test_fp16_encoder_matches_numpy():
    rng = np.random.default_rng(2)
    h = np.arange(65536, dtype=np.uint16).view(np.float16)
    fin = h[np.isfinite(h)].astype(np.float32)
    mids = []
    hs = np.sort(np.unique(np.abs(fin.astype(np.float64))))
    mids = ((hs[1:] + hs[:-1]) / 2).astype(np.float32)
    x = np.concatenate([fin, mids, np.nextafter(mids, np.float32(np.inf)),
                        np.nextafter(mids, np.float32(0)),
                        rng.standard_normal(100000).astype(np.float32) * 100,
                        np.array([65519.0, 65520.0, 7e4, 1e-8, 2 ** -25, 3 * 2 ** -26], np.float32)])
    x = np.concatenate([x, -x])
    ours = oracle.encode_fp16(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]
    codes = np.arange(65536, dtype=np.uint16)
    dec = oracle.decode_fp16(codes)
    ref = codes.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert (np.isnan(dec) == nan).all() and (dec[~nan] == ref[~nan]).all()
