"""Pins for the oracle's paged decode attention.

Checked against: brute force with Python floats on tiny inputs (no paging),
PyTorch's fp64 scaled_dot_product_attention on the gathered KV (library
routine), closed forms (constant keys, one token, two tokens, sharpened
softmax), and the invariants the PagedAttention description fixes: outputs do
not depend on which physical blocks hold the data, and a block shared by several
tables gives the same result as private copies.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import brute_force_attention, random_tables, slots, to_f64

DTS = [oracle.DT_FP16, oracle.DT_BF16, oracle.DT_E4M3, oracle.DT_E5M2, oracle.DT_E2M1]


def build(rng, dt, lens, H, D, nb, q_heads, bt=None, kv=None, in_dtype=torch.bfloat16):
    if dt == oracle.DT_FP16:
        in_dtype = torch.float16
    if bt is None:
        bt = random_tables(rng, lens, nb)
    c = oracle.Cache(dt, nb, H, D)
    kvs = []
    for b, L in enumerate(lens):
        if kv is not None:
            k, v = kv[b]
        else:
            k = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(in_dtype)
            v = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(in_dtype)
        kvs.append((k, v))
        if L:
            assert oracle.kv_cache_write(c, k, v, slots(bt[b], 0, L)) == 0
    qd = torch.float16 if dt == oracle.DT_FP16 else torch.bfloat16
    q = torch.from_numpy(rng.standard_normal((len(lens), q_heads, D), dtype=np.float32)).to(qd)
    return c, bt, kvs, q


def test_brute_force_tiny_16bit():
    rng = np.random.default_rng(10)
    for dt in (oracle.DT_FP16, oracle.DT_BF16):
        lens = [1, 17, 40]
        c, bt, kvs, q = build(rng, dt, lens, 2, 64, 16, 4)
        out, err = oracle.paged_decode(c, q, bt, np.array(lens, np.int32), 0.125)
        assert err == 0
        for b, L in enumerate(lens):
            k, v = kvs[b]
            for hq in range(4):
                h = hq // 2
                ref = brute_force_attention(to_f64(q[b, hq]).tolist(), to_f64(k[:, h]).tolist(),
                                            to_f64(v[:, h]).tolist(), 0.125)
                np.testing.assert_allclose(out[b, hq], ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("dt", DTS)
def test_matches_torch_sdpa_on_gathered_kv(dt):
    rng = np.random.default_rng(11 + dt)
    lens = [5, 16, 33, 70]
    H, G, D = 2, 3, 64
    c, bt, kvs, q = build(rng, dt, lens, H, D, 40, H * G)
    scale = float(np.float32(0.1))  # the oracle takes the scale as float32
    out, err = oracle.paged_decode(c, q, bt, np.array(lens, np.int32), scale)
    assert err == 0
    for b, L in enumerate(lens):
        for h in range(H):
            kd, vd, valid = oracle.gather(c, bt[b], L, h)
            assert valid.all()
            qq = torch.from_numpy(to_f64(q[b, h * G:(h + 1) * G]))[None]           # [1,G,D]
            kk = torch.from_numpy(kd)[None, None].expand(1, G, L, D)
            vv = torch.from_numpy(vd)[None, None].expand(1, G, L, D)
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[:, :, None, :].reshape(1, G, 1, D), kk, vv, scale=scale)[0, :, 0].numpy()
            np.testing.assert_allclose(out[b, h * G:(h + 1) * G], ref, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("dt", DTS)
def test_closed_form_constant_keys_give_mean_of_values(dt):
    rng = np.random.default_rng(20 + dt)
    L, H, D = 37, 1, 64
    row = rng.standard_normal(D).astype(np.float32)
    ind = torch.float16 if dt == oracle.DT_FP16 else torch.bfloat16
    k = torch.from_numpy(np.tile(row, (L, H, 1))).to(ind)
    v = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(ind)
    c, bt, _, q = build(rng, dt, [L], H, D, 8, 2, kv=[(k, v)])
    out, _ = oracle.paged_decode(c, q, bt, np.array([L], np.int32), 0.3)
    _, vd, _ = oracle.gather(c, bt[0], L, 0)
    for hq in range(2):
        np.testing.assert_allclose(out[0, hq], vd.mean(axis=0), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("dt", DTS)
def test_closed_forms_one_and_two_tokens(dt):
    rng = np.random.default_rng(30 + dt)
    H, D = 1, 64
    c, bt, _, q = build(rng, dt, [1, 2], H, D, 8, 1)
    scale = 0.25
    out, _ = oracle.paged_decode(c, q, bt, np.array([1, 2], np.int32), scale)
    _, v0, _ = oracle.gather(c, bt[0], 1, 0)
    np.testing.assert_array_equal(out[0, 0], v0[0])
    k1, v1, _ = oracle.gather(c, bt[1], 2, 0)
    qd = to_f64(q[1, 0])
    ds = scale * (qd @ k1[1] - qd @ k1[0])
    w1 = 1.0 / (1.0 + math.exp(-ds))
    np.testing.assert_allclose(out[1, 0], w1 * v1[1] + (1 - w1) * v1[0], rtol=1e-12, atol=1e-14)


def test_sharpened_softmax_tends_to_argmax():
    rng = np.random.default_rng(40)
    L, D = 50, 64
    c, bt, kvs, q = build(rng, oracle.DT_BF16, [L], 1, D, 8, 1)
    q_big = (q.float() * 100).to(torch.bfloat16)
    out, _ = oracle.paged_decode(c, q_big, bt, np.array([L], np.int32), 1.0)
    k, v = kvs[0]
    s = to_f64(k[:, 0]) @ to_f64(q_big[0, 0])
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out[0, 0], to_f64(v[:, 0])[np.argmax(s)], atol=1e-6)


@pytest.mark.parametrize("dt", DTS)
def test_physical_block_permutation_is_invisible(dt):
    rng = np.random.default_rng(50 + dt)
    lens = [20, 47, 64, 3]
    H, D, nb = 2, 64, 64
    c1, bt1, kvs, q = build(rng, dt, lens, H, D, nb, 4)
    perm = rng.permutation(nb).astype(np.int32)
    bt2 = np.where(bt1 >= 0, perm[np.maximum(bt1, 0)], -1).astype(np.int32)
    c2, _, _, _ = build(rng, dt, lens, H, D, nb, 4, bt=bt2, kv=kvs)
    o1, _ = oracle.paged_decode(c1, q, bt1, np.array(lens, np.int32), 0.125)
    o2, _ = oracle.paged_decode(c2, q, bt2, np.array(lens, np.int32), 0.125)
    np.testing.assert_array_equal(o1, o2)


@pytest.mark.parametrize("dt", DTS)
def test_shared_prefix_equals_private_copies(dt):
    rng = np.random.default_rng(60 + dt)
    H, D, nb = 2, 64, 64
    P = 32  # two full blocks
    lens = [P + 10, P + 25, P + 3]
    ind = torch.float16 if dt == oracle.DT_FP16 else torch.bfloat16
    pk = torch.from_numpy(rng.standard_normal((P, H, D), dtype=np.float32)).to(ind)
    pv = torch.from_numpy(rng.standard_normal((P, H, D), dtype=np.float32)).to(ind)
    kvs = []
    for L in lens:
        k = torch.cat([pk, torch.from_numpy(rng.standard_normal((L - P, H, D), dtype=np.float32)).to(ind)])
        v = torch.cat([pv, torch.from_numpy(rng.standard_normal((L - P, H, D), dtype=np.float32)).to(ind)])
        kvs.append((k, v))
    _, _, _, q = build(rng, dt, lens, H, D, nb, 4, kv=kvs)
    bt_priv = random_tables(rng, lens, nb)
    c_priv, _, _, _ = build(rng, dt, lens, H, D, nb, 4, bt=bt_priv, kv=kvs)
    bt_sh = random_tables(rng, lens, nb, shared_prefix_blocks=2, n_share=3)
    c_sh = oracle.Cache(dt, nb, H, D)
    for b, L in enumerate(lens):
        lo = 0 if b == 0 else P  # the prefix is written once
        oracle.kv_cache_write(c_sh, kvs[b][0][lo:], kvs[b][1][lo:], slots(bt_sh[b], lo, L - lo))
    o1, _ = oracle.paged_decode(c_priv, q, bt_priv, np.array(lens, np.int32), 0.125)
    o2, _ = oracle.paged_decode(c_sh, q, bt_sh, np.array(lens, np.int32), 0.125)
    np.testing.assert_array_equal(o1, o2)


@pytest.mark.parametrize("dt", DTS)
def test_poison_never_reaches_outputs(dt):
    rng = np.random.default_rng(70 + dt)
    lens = [1, 15, 17, 31]
    c, bt, _, q = build(rng, dt, lens, 2, 64, 32, 4)
    out, err = oracle.paged_decode(c, q, bt, np.array(lens, np.int32), 0.125)
    assert err == 0 and np.all(np.isfinite(out))


def test_error_cases():
    rng = np.random.default_rng(80)
    lens = [20, 20, 20]
    c, bt, _, q = build(rng, oracle.DT_BF16, lens, 2, 64, 16, 4)
    out, err = oracle.paged_decode(c, q, bt, np.array([0, 20, 20], np.int32), 0.125)
    assert err == 0 and not out[0].any() and out[1].any()
    out, err = oracle.paged_decode(c, q, bt, np.array([20, 16 * bt.shape[1] + 1, 20], np.int32), 0.125)
    assert err == oracle.ERR_SEQ_LEN and not out[1].any() and out[0].any()
    bad = bt.copy()
    bad[2, 1] = 999
    out, err = oracle.paged_decode(c, q, bad, np.array(lens, np.int32), 0.125)
    assert err == oracle.ERR_BLOCK_ID
    # the sequence keeps its first (valid) block
    ok, _ = oracle.paged_decode(c, q, bt, np.array([20, 20, 16], np.int32), 0.125)
    np.testing.assert_allclose(out[2], ok[2], rtol=1e-12)
