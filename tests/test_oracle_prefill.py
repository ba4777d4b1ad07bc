"""Pins of the oracle's chunked-prefill attention ("vLLM" glossary, "Chunked
prefill"; the compression article's architecture diagram processes prompts in
512-token chunks): brute force with Python floats on contiguous K/V, the
single-query case against the oracle's decode, the causal property (a query
never sees later positions) and the rejection of a chunk longer than its
sequence."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import brute_force_attention, random_tables, slots, to_f64


def _setup(dt, lens, qlens, H=2, Hq=4, D=64, seed=0):
    rng = np.random.default_rng(seed)
    nb = sum((L + 15) // 16 for L in lens) + 3
    bt = random_tables(rng, lens, nb)
    c = oracle.Cache(dt, nb, H, D)
    tdt = torch.float16 if dt == oracle.DT_FP16 else torch.bfloat16
    kv = []
    for b, L in enumerate(lens):
        k = torch.from_numpy(rng.standard_normal((L, H, D)).astype(np.float32)).to(tdt)
        v = torch.from_numpy(rng.standard_normal((L, H, D)).astype(np.float32)).to(tdt)
        assert oracle.kv_cache_write(c, k, v, slots(bt[b], 0, L)) == 0
        kv.append((k, v))
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.from_numpy(rng.standard_normal((int(cu[-1]), Hq, D)).astype(np.float32)).to(tdt)
    return rng, c, bt, kv, cu, q


def test_prefill_matches_brute_force_on_contiguous_kv():
    lens, qlens = [37, 20], [5, 20]
    H, Hq, D = 2, 4, 64
    _, c, bt, kv, cu, q = _setup(oracle.DT_BF16, lens, qlens, H, Hq, D)
    scale = 0.125
    out, err = oracle.paged_prefill(c, q, cu, bt, np.array(lens, np.int32), scale)
    assert err == 0
    G = Hq // H
    for b, L in enumerate(lens):
        kf, vf = to_f64(kv[b][0]), to_f64(kv[b][1])
        for i in range(qlens[b]):
            pos = L - qlens[b] + i
            for hq in range(Hq):
                h = hq // G
                want = brute_force_attention(to_f64(q[cu[b] + i, hq]), kf[:pos + 1, h], vf[:pos + 1, h], scale)
                np.testing.assert_allclose(out[cu[b] + i, hq], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dt", [oracle.DT_FP16, oracle.DT_E4M3, oracle.DT_E2M1])
def test_each_prefill_row_equals_decode_at_its_position(dt):
    lens, qlens = [50, 33, 16], [7, 1, 16]
    _, c, bt, _, cu, q = _setup(dt, lens, qlens, seed=1)
    out, err = oracle.paged_prefill(c, q, cu, bt, np.array(lens, np.int32), 0.1)
    assert err == 0
    for b, L in enumerate(lens):
        for i in range(qlens[b]):
            pos = L - qlens[b] + i
            one, e = oracle.paged_decode(c, q[cu[b] + i][None], bt[b:b + 1], np.array([pos + 1], np.int32), 0.1)
            assert e == 0
            np.testing.assert_array_equal(out[cu[b] + i], one[0])


def test_a_query_never_sees_later_positions():
    lens, qlens = [48], [12]
    _, c, bt, _, cu, q = _setup(oracle.DT_BF16, lens, qlens, seed=2)
    out, _ = oracle.paged_prefill(c, q, cu, bt, np.array(lens, np.int32), 0.1)
    # overwrite the K/V of the last 4 positions (44..47) with other values
    k2 = torch.full((4, 2, 64), 3.0, dtype=torch.bfloat16)
    oracle.kv_cache_write(c, k2, -k2, slots(bt[0], 44, 4))
    out2, _ = oracle.paged_prefill(c, q, cu, bt, np.array(lens, np.int32), 0.1)
    # query tokens 0..7 sit at positions 36..43: unchanged; 8..11 see the new K/V
    np.testing.assert_array_equal(out[:8], out2[:8])
    assert (np.abs(out[8:] - out2[8:]) > 1e-6).any(axis=(1, 2)).all()


def test_chunk_longer_than_its_sequence_is_rejected():
    lens, qlens = [10, 20], [11, 3]
    _, c, bt, _, cu, q = _setup(oracle.DT_BF16, [10, 20], [11, 3], seed=3)
    out, err = oracle.paged_prefill(c, q, cu, bt, np.array(lens, np.int32), 0.1)
    assert err == oracle.ERR_SEQ_LEN
    assert (out[:11] == 0).all() and (np.abs(out[11:]) > 0).any()
