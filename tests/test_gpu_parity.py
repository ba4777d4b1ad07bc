"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Cache bytes (codes, scales, outlier buffers, untouched poison) must match bit
for bit; attention outputs must lie within atol + rtol * |ref| of the fp64
oracle (2e-3 + 1e-2 for 16-bit and FP8 caches, 5e-3 + 1e-2 for FP4).
Sizes span several blocks, splits and ragged tails.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh
from tests.helpers import random_tables, slots

pytestmark = pytest.mark.gpu

pq = pytest.importorskip("paged_quantized_kv_cache_b200")

CASES = [
    # kv_dtype, q dtype, D, Hq, Hkv
    (pq.FP16, torch.float16, 64, 8, 2),
    (pq.BF16, torch.bfloat16, 128, 32, 8),
    (pq.BF16, torch.bfloat16, 64, 8, 8),
    (pq.FP8_E4M3, torch.bfloat16, 128, 32, 8),
    (pq.FP8_E4M3, torch.float16, 64, 16, 2),
    (pq.FP8_E5M2, torch.bfloat16, 128, 8, 1),
    (pq.FP4_E2M1, torch.bfloat16, 128, 32, 8),
    (pq.FP4_E2M1, torch.float16, 64, 8, 4),
]


def _kv(rng, L, H, D, dtype, outliers=False):
    x = rng.standard_normal((L, H, D)).astype(np.float32)
    y = rng.standard_normal((L, H, D)).astype(np.float32)
    if outliers:
        for h in range(H):
            x[:, h, rng.choice(D, 2, replace=False)] *= 16
            y[:, h, rng.choice(D, 2, replace=False)] *= 16
    return torch.from_numpy(x).to(dtype), torch.from_numpy(y).to(dtype)


def _scenario(case, lens, seed, chunk=None, nb_extra=7):
    kv_dtype, qdt, D, Hq, Hkv = case
    rng = np.random.default_rng(seed)
    nb = sum((L + 15) // 16 for L in lens) + nb_extra
    bt = random_tables(rng, lens, nb)
    g, o = gh.new_pair(kv_dtype, nb, Hkv, D)
    kvs = [_kv(rng, L, Hkv, D, qdt, outliers=(kv_dtype == pq.FP4_E2M1)) for L in lens]
    if chunk is None:
        for b, L in enumerate(lens):
            if L:
                ge, oe = gh.write_both(g, o, kvs[b][0], kvs[b][1], slots(bt[b], 0, L))
                assert ge == oe == 0
    else:
        # chunked writes across all sequences: blocks get appended to
        for lo in range(0, max(lens), chunk):
            ks, vs, ss = [], [], []
            for b, L in enumerate(lens):
                hi = min(L, lo + chunk)
                if hi > lo:
                    ks.append(kvs[b][0][lo:hi]); vs.append(kvs[b][1][lo:hi])
                    ss.append(slots(bt[b], lo, hi - lo))
            ge, oe = gh.write_both(g, o, torch.cat(ks), torch.cat(vs), np.concatenate(ss))
            assert ge == oe == 0
    q = torch.from_numpy(rng.standard_normal((len(lens), Hq, D)).astype(np.float32)).to(qdt)
    return g, o, bt, q


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-D%d-G%d" % (pq.DTYPE_NAMES[c[0]], c[2], c[3] // c[4]))
@pytest.mark.parametrize("split", [0, 3])
def test_write_and_decode_match_oracle(case, split):
    lens = [1, 15, 16, 17, 33, 100, 250, 513]
    g, o, bt, q = _scenario(case, lens, seed=100 + case[0])
    gh.assert_cache_equal(g, o, tag="prefill")
    scale = float(np.float32(1.0 / np.sqrt(case[2])))
    out, err = gh.decode_gpu(g, q, bt, lens, scale, split_blocks=split)
    ref, oerr = oracle.paged_decode(o, q, bt, np.array(lens, np.int32), scale)
    assert err == 0 and oerr == 0
    assert torch.isfinite(out).all()
    gh.assert_close(out, ref, case[0], tag=str(case))


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-D%d" % (pq.DTYPE_NAMES[c[0]], c[2]))
def test_chunked_appends_match_oracle(case):
    # 40-token chunks start runs in the middle of blocks: FP8 scales grow and
    # re-encode, FP4 reuses the outlier set chosen at the block's first write
    lens = [3, 40, 57, 130, 200]
    g, o, bt, q = _scenario(case, lens, seed=200 + case[0], chunk=40)
    gh.assert_cache_equal(g, o, tag="chunked")
    scale = 0.1
    out, _ = gh.decode_gpu(g, q, bt, lens, scale)
    ref, _ = oracle.paged_decode(o, q, bt, np.array(lens, np.int32), scale)
    gh.assert_close(out, ref, case[0], tag="chunked " + str(case))


@pytest.mark.parametrize("kv_dtype", [pq.FP8_E4M3, pq.FP8_E5M2, pq.FP4_E2M1, pq.BF16])
def test_single_token_appends(kv_dtype):
    # decode-time writes: one new token per sequence per call
    case = next(c for c in CASES if c[0] == kv_dtype)
    _, qdt, D, Hq, Hkv = case
    rng = np.random.default_rng(7)
    lens = [5, 16, 31, 64]
    nb = 32
    bt = random_tables(rng, [L + 6 for L in lens], nb)
    g, o = gh.new_pair(kv_dtype, nb, Hkv, D)
    kvs = [_kv(rng, L + 6, Hkv, D, qdt) for L in lens]
    for b, L in enumerate(lens):
        gh.write_both(g, o, kvs[b][0][:L], kvs[b][1][:L], slots(bt[b], 0, L))
    for step in range(6):
        k = torch.stack([kvs[b][0][L + step] for b, L in enumerate(lens)])
        v = torch.stack([kvs[b][1][L + step] for b, L in enumerate(lens)])
        # later steps grow the values so FP8 scales must grow on append
        k = (k.float() * (1 + step)).to(qdt)
        v = (v.float() * (1 + step)).to(qdt)
        s = np.array([slots(bt[b], L + step, 1)[0] for b, L in enumerate(lens)], np.int32)
        ge, oe = gh.write_both(g, o, k, v, s)
        assert ge == oe == 0
        gh.assert_cache_equal(g, o, tag="append step %d" % step)
    q = torch.from_numpy(rng.standard_normal((len(lens), Hq, D)).astype(np.float32)).to(qdt)
    L2 = [L + 6 for L in lens]
    out, _ = gh.decode_gpu(g, q, bt, L2, 0.125)
    ref, _ = oracle.paged_decode(o, q, bt, np.array(L2, np.int32), 0.125)
    gh.assert_close(out, ref, kv_dtype)


@pytest.mark.parametrize("case", CASES[:1] + CASES[3:4] + CASES[6:7], ids=lambda c: pq.DTYPE_NAMES[c[0]])
def test_block_permutation_and_sharing_are_bit_identical_on_gpu(case):
    kv_dtype, qdt, D, Hq, Hkv = case
    rng = np.random.default_rng(300)
    P = 48
    lens = [P + 5, P + 37, P + 16]
    pk, pv = _kv(rng, P, Hkv, D, qdt)
    kvs = []
    for L in lens:
        k, v = _kv(rng, L - P, Hkv, D, qdt)
        kvs.append((torch.cat([pk, k]), torch.cat([pv, v])))
    q = torch.from_numpy(rng.standard_normal((3, Hq, D)).astype(np.float32)).to(qdt)
    nb = 64
    outs = []
    for variant in range(3):
        if variant < 2:
            bt = random_tables(rng, lens, nb)
            g = pq.allocate_cache(kv_dtype, nb, Hkv, D, fill=0xFF)
            for b, L in enumerate(lens):
                pq.kv_cache_write(kvs[b][0].cuda(), kvs[b][1].cuda(),
                                  torch.from_numpy(slots(bt[b], 0, L)).cuda(), g, gh.err_flag())
        else:
            bt = random_tables(rng, lens, nb, shared_prefix_blocks=3, n_share=3)
            g = pq.allocate_cache(kv_dtype, nb, Hkv, D, fill=0xFF)
            for b, L in enumerate(lens):
                lo = 0 if b == 0 else P
                pq.kv_cache_write(kvs[b][0][lo:].cuda(), kvs[b][1][lo:].cuda(),
                                  torch.from_numpy(slots(bt[b], lo, L - lo)).cuda(), g, gh.err_flag())
        out, err = gh.decode_gpu(g, q, bt, lens, 0.125)
        assert err == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-D%d" % (pq.DTYPE_NAMES[c[0]], c[2]))
def test_split_size_changes_only_rounding(case):
    lens = [700, 1, 333, 64]
    g, o, bt, q = _scenario(case, lens, seed=400 + case[0])
    outs = [gh.decode_gpu(g, q, bt, lens, 0.09, split_blocks=s)[0] for s in (0, 1, 5, 32, 1000)]
    ref, _ = oracle.paged_decode(o, q, bt, np.array(lens, np.int32), 0.09)
    for out in outs:
        gh.assert_close(out, ref, case[0])
        atol, rtol = gh.TOL[case[0]]
        assert torch.allclose(out.float(), outs[0].float(), atol=atol, rtol=rtol)


def test_repeated_calls_are_deterministic_and_reuse_the_workspace():
    case = CASES[1]
    lens = [900, 17, 2000, 5]
    g, o, bt, q = _scenario(case, lens, seed=500)
    bt_d = torch.from_numpy(bt).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = pq.decode_workspace(len(lens), case[3], case[4], case[2], bt.shape[1])
    qd = q.cuda()
    first = None
    for it in range(5):
        out = torch.empty_like(qd)
        e = gh.err_flag()
        if it == 3:
            ws.fill_(0xAB)  # results do not depend on what the workspace held
        pq.paged_decode_attention(qd, g, bt_d, sl, 0.1, out, ws, e)
        if first is None:
            first = out
        assert torch.equal(out, first) and int(e.item()) == 0


def test_arrival_words_left_by_other_split_plans_do_not_matter():
    """Split pairs are merged by the warp whose piece arrives last, counted in
    per-chunk words of the workspace tagged with the launch. One workspace
    serves calls with different split plans in turn (so words written under one
    plan lie under the chunks of the next); every result equals the same call
    on a fresh zeroed workspace, bit for bit."""
    case = CASES[4]
    lens = [1200, 17, 700, 5, 333]
    g, o, bt, q = _scenario(case, lens, seed=510)
    bt_d = torch.from_numpy(bt).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    qd = q.cuda()
    plans = (1, 5, 0, 3, 1, 0, 7, 1)
    shared = torch.zeros(max(pq.decode_workspace_bytes(len(lens), case[3], case[4], case[2], bt.shape[1], s)
                             for s in plans), dtype=torch.uint8, device="cuda")
    for split in plans:
        need = pq.decode_workspace_bytes(len(lens), case[3], case[4], case[2], bt.shape[1], split)
        fresh = torch.zeros(need, dtype=torch.uint8, device="cuda")
        a, b = torch.empty_like(qd), torch.empty_like(qd)
        e1, e2 = gh.err_flag(), gh.err_flag()
        pq.paged_decode_attention(qd, g, bt_d, sl, 0.1, a, shared, e1, split_blocks=split)
        pq.paged_decode_attention(qd, g, bt_d, sl, 0.1, b, fresh, e2, split_blocks=split)
        torch.cuda.synchronize()
        assert int(e1.item()) == int(e2.item()) == 0
        assert torch.equal(a, b), "split %d" % split
    ref, _ = oracle.paged_decode(o, q, bt, np.array(lens, np.int32), 0.1)
    gh.assert_close(a, ref, case[0])


def test_partial_floats_left_in_a_workspace_are_never_read_as_arrival_words():
    """A workspace reused with another layout has its arrival words where
    partial outputs were: float pairs such as (+0.0 above 1.0f) or a -inf row
    maximum. Launch tags start with the byte 0xFF and use a 31-bit counter, so
    no such word is taken for a tag: every call on a workspace filled with
    these patterns equals the same call on a fresh one, bit for bit."""
    case = CASES[4]
    lens = [1200, 17, 700, 5, 333]
    g, o, bt, q = _scenario(case, lens, seed=511)
    bt_d = torch.from_numpy(bt).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    qd = q.cuda()
    pairs = [(0.0, 1.0), (float("-inf"), 0.0), (float("-inf"), float("-inf")), (0.5, -2.0), (-0.0, 3.0e38)]
    for split in (1, 3, 0):
        need = pq.decode_workspace_bytes(len(lens), case[3], case[4], case[2], bt.shape[1], split)
        fresh = torch.zeros(need, dtype=torch.uint8, device="cuda")
        b = torch.empty_like(qd)
        e2 = gh.err_flag()
        pq.paged_decode_attention(qd, g, bt_d, sl, 0.1, b, fresh, e2, split_blocks=split)
        for lo, hi in pairs:
            words = torch.tensor([lo, hi], dtype=torch.float32).repeat((need + 7) // 8)
            ws = words.view(torch.uint8)[:need].clone().cuda()
            a = torch.empty_like(qd)
            e1 = gh.err_flag()
            pq.paged_decode_attention(qd, g, bt_d, sl, 0.1, a, ws, e1, split_blocks=split)
            torch.cuda.synchronize()
            assert int(e1.item()) == int(e2.item()) == 0
            assert torch.equal(a, b), "split %d, words (%r, %r)" % (split, lo, hi)


def test_edge_lengths_and_error_bits():
    case = CASES[1]
    kv_dtype, qdt, D, Hq, Hkv = case
    lens = [0, 1, 16, 17, 48]
    g, o, bt, q = _scenario(case, lens, seed=600)
    out, err = gh.decode_gpu(g, q, bt, lens, 0.1)
    assert err == 0
    assert torch.count_nonzero(out[0]) == 0
    ref, _ = oracle.paged_decode(o, q, bt, np.array(lens, np.int32), 0.1)
    gh.assert_close(out, ref, kv_dtype)
    # L = 1 returns v_0 (up to the output rounding)
    kd, vd, _ = oracle.gather(o, bt[1], 1, 0)
    assert np.allclose(out[1, 0].double().cpu().numpy(), vd[0], atol=1e-2, rtol=1e-2)
    # seq_len past the table: error bit, zero rows; others unaffected
    bad_lens = list(lens)
    bad_lens[2] = 16 * bt.shape[1] + 1
    out2, err2 = gh.decode_gpu(g, q, bt, bad_lens, 0.1)
    assert err2 & pq.DEVERR_SEQ_LEN
    assert torch.count_nonzero(out2[2]) == 0
    assert torch.equal(out2[4], out[4])
    # a table entry outside the pool: error bit, block skipped, no NaN
    bt3 = bt.copy()
    bt3[4, 1] = g.num_blocks + 5
    out3, err3 = gh.decode_gpu(g, q, bt3, lens, 0.1)
    assert err3 & pq.DEVERR_BLOCK_ID and torch.isfinite(out3).all()
    ref3, _ = oracle.paged_decode(o, q, bt3, np.array(lens, np.int32), 0.1)
    gh.assert_close(out3, ref3, kv_dtype)


@pytest.mark.parametrize("kv_dtype", [pq.BF16, pq.FP8_E4M3, pq.FP4_E2M1])
def test_write_error_bits_match_oracle(kv_dtype):
    case = next(c for c in CASES if c[0] == kv_dtype)
    _, qdt, D, Hq, Hkv = case
    g, o = gh.new_pair(kv_dtype, 4, Hkv, D)
    rng = np.random.default_rng(8)
    k, v = _kv(rng, 4, Hkv, D, qdt)
    # token 1 points past the pool: skipped and flagged; the others are written
    ge, oe = gh.write_both(g, o, k, v, np.array([0, 4 * 16 + 3, -1, 16], np.int32))
    assert ge == oe and ge & pq.DEVERR_SLOT
    gh.assert_cache_equal(g, o, tag="slot error")
    if kv_dtype != pq.BF16:
        # two adjacent tokens in one block with a gap in their offsets: flagged
        # (their order in the block is unspecified, so no bytes are compared)
        ge, oe = gh.write_both(g, o, k[:2], v[:2], np.array([36, 39], np.int32))
        assert ge & pq.DEVERR_RUN and oe & pq.DEVERR_RUN
    # empty call is a no-op
    pq.kv_cache_write(k[:0].cuda(), v[:0].cuda(), torch.zeros(0, dtype=torch.int32, device="cuda"), g,
                      gh.err_flag())


def test_tiny_workload_end_to_end():
    """The 4-sequence fp16 workload (lens 17, 33, 64, 100; 8 q / 2 KV heads; D 64;
    tables = one permutation of a 64-block pool), in full."""
    import workloads as W
    s = W.spec("tiny")
    tab = W.tables(s)
    g, o = gh.new_pair(s.kv_dtype, tab.num_blocks, s.num_kv_heads, s.head_dim)
    for call in W.prefill_calls(s):
        k, v, sl = W.gather_call(s, call, tab)
        ge, oe = gh.write_both(g, o, k, v, sl)
        assert ge == oe == 0
    gh.assert_cache_equal(g, o)
    q = W.query(s)
    lens = W.decode_lens(s)
    out, err = gh.decode_gpu(g, q, tab.block_tables, lens, W.softmax_scale(s))
    ref, _ = oracle.paged_decode(o, q, tab.block_tables, lens, W.softmax_scale(s))
    assert err == 0
    gh.assert_close(out, ref, s.kv_dtype)
