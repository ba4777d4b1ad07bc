"""GPU parity of the chunked-prefill attention (tcgen05 kernel) against the
oracle ("vLLM" glossary, "Chunked prefill"; the compression article's
architecture diagram: 512-token chunks, the attention kernel reading codes and
fp16 outliers together).

Sequences mix chunks that span several 128-row query tiles with a ragged last
tile, a chunk that is the whole sequence (causal from position 0), a
single-token chunk, and KV lengths that end inside a block; outputs must lie
within atol + rtol * |ref| of the fp64 oracle (2e-3 + 1e-2 for 16-bit and FP8
caches, 5e-3 + 1e-2 for FP4)."""
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
    (pq.BF16, torch.bfloat16, 128, 32, 8),
    (pq.FP16, torch.float16, 64, 8, 2),
    (pq.BF16, torch.bfloat16, 64, 8, 8),
    (pq.BF16, torch.bfloat16, 128, 64, 8),
    (pq.FP8_E4M3, torch.bfloat16, 128, 32, 8),
    (pq.FP8_E5M2, torch.float16, 64, 16, 2),
    (pq.FP4_E2M1, torch.bfloat16, 128, 32, 8),
    (pq.FP4_E2M1, torch.float16, 64, 8, 4),
]


def _build(case, lens, qlens, seed, bad_block=None, extra=5):
    kv_dtype, qdt, D, Hq, Hkv = case
    rng = np.random.default_rng(seed)
    nb = sum((L + 15) // 16 for L in lens) + extra
    bt = random_tables(rng, lens, nb)
    g, o = gh.new_pair(kv_dtype, nb, Hkv, D)
    in_dt = torch.float16 if qdt == torch.float16 else torch.bfloat16
    for b, L in enumerate(lens):
        k = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        v = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        if kv_dtype == pq.FP4_E2M1:
            for h in range(Hkv):
                k[:, h, rng.choice(D, 2, replace=False)] *= 16
                v[:, h, rng.choice(D, 2, replace=False)] *= 16
        kt, vt = torch.from_numpy(k).to(in_dt), torch.from_numpy(v).to(in_dt)
        ge, oe = gh.write_both(g, o, kt, vt, slots(bt[b], 0, L))
        assert ge == oe == 0
    gh.assert_cache_equal(g, o, tag="prefill setup")
    if bad_block is not None:
        b, j = bad_block
        bt = bt.copy()
        bt[b, j] = nb + 3
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.from_numpy(rng.standard_normal((int(cu[-1]), Hq, D)).astype(np.float32)).to(qdt)
    return g, o, bt, cu, q


def _run(g, q, cu, bt, lens, scale, max_q_len=None):
    B = len(lens)
    out = torch.full_like(q.cuda(), float("nan"))
    e = gh.err_flag()
    mq = int(max(np.diff(cu))) if max_q_len is None else max_q_len
    pq.paged_prefill_attention(q.cuda(), torch.from_numpy(cu).cuda(), max(1, mq), g,
                               torch.from_numpy(np.ascontiguousarray(bt, np.int32)).cuda(),
                               torch.from_numpy(np.array(lens, np.int32)).cuda(), scale, out, e)
    torch.cuda.synchronize()
    return out, int(e.item())


@pytest.mark.parametrize("case", CASES, ids=lambda c: "kv%d-D%d-G%d" % (c[0], c[2], c[3] // c[4]))
def test_prefill_matches_oracle(case):
    lens = [700, 64, 301, 97]
    qlens = [200, 64, 1, 33]
    D = case[2]
    g, o, bt, cu, q = _build(case, lens, qlens, seed=40 + case[0])
    scale = 1.0 / np.sqrt(D)
    out, err = _run(g, q, cu, bt, lens, scale)
    ref, rerr = oracle.paged_prefill(o, q, cu, bt, np.array(lens, np.int32), scale)
    assert err == rerr == 0
    gh.assert_close(out, ref, case[0], tag="prefill")


@pytest.mark.parametrize("case", [CASES[0], CASES[4], CASES[6]], ids=["bf16", "fp8", "fp4"])
def test_prefill_long_context_512_token_chunk(case):
    """A 512-token chunk after a 1500-token prefix: 16 query tiles (G = 4), 32 KV tiles."""
    lens, qlens = [2012, 520], [512, 8]
    g, o, bt, cu, q = _build(case, lens, qlens, seed=50)
    out, err = _run(g, q, cu, bt, lens, 0.088)
    ref, rerr = oracle.paged_prefill(o, q, cu, bt, np.array(lens, np.int32), 0.088)
    assert err == rerr == 0
    gh.assert_close(out, ref, case[0], tag="prefill 512")


def test_prefill_edge_cases_and_error_bits():
    case = CASES[1]
    # sequence 1: chunk longer than the sequence (zero rows, SEQ_LEN);
    # sequence 2: empty chunk; sequence 3: one block id out of range (skipped)
    lens, qlens = [40, 5, 30, 50], [10, 8, 0, 20]
    g, o, bt, cu, q = _build(case, lens, qlens, seed=60, bad_block=(3, 1))
    out, err = _run(g, q, cu, bt, lens, 0.125)
    ref, rerr = oracle.paged_prefill(o, q, cu, bt, np.array(lens, np.int32), 0.125)
    assert err == rerr == pq.DEVERR_SEQ_LEN | pq.DEVERR_BLOCK_ID
    assert torch.all(out[10:18] == 0)
    gh.assert_close(out, ref, case[0], tag="prefill edges")


def test_prefill_rows_past_max_q_len_are_flagged():
    case = CASES[1]
    lens, qlens = [100], [40]
    g, o, bt, cu, q = _build(case, lens, qlens, seed=61)
    out, err = _run(g, q, cu, bt, lens, 0.125, max_q_len=16)  # G = 4: one tile of 32 tokens
    assert err == pq.DEVERR_SEQ_LEN
    ref, _ = oracle.paged_prefill(o, q, cu, bt, np.array(lens, np.int32), 0.125)
    gh.assert_close(out[:32], ref[:32], case[0], tag="computed rows")


def test_prefill_is_deterministic_and_layout_invariant():
    case = CASES[4]
    lens, qlens = [300, 130], [130, 130]
    g, o, bt, cu, q = _build(case, lens, qlens, seed=62, extra=24)
    a, _ = _run(g, q, cu, bt, lens, 0.09)
    b, _ = _run(g, q, cu, bt, lens, 0.09)
    assert torch.equal(a, b)
    # move every block of sequence 0 to other ids: the same bits come out
    nb = g.num_blocks
    used = set(int(x) for x in bt.ravel() if x >= 0)
    free = [i for i in range(nb) if i not in used]
    n0 = (lens[0] + 15) // 16
    assert len(free) >= n0
    pairs = np.stack([bt[0, :n0], free[:n0]], axis=1).astype(np.int32)
    e = gh.err_flag()
    pq.copy_blocks(g, torch.from_numpy(pairs).cuda(), e)
    bt2 = bt.copy()
    bt2[0, :n0] = free[:n0]
    c, _ = _run(g, q, cu, bt2, lens, 0.09)
    assert torch.equal(a, c)


@pytest.mark.parametrize("case", [CASES[0], CASES[4], CASES[6]], ids=["bf16", "fp8", "fp4"])
def test_prefill_wait_limit_runs_out_and_the_next_call_is_correct(case):
    """With a 1 ns limit, the prefill's waits (on its copies, its tensor-core
    products and the other warps) give up while the work is still on the way:
    the call reports PQKV_DEVERR_TIMEOUT, lets every copy and product in flight
    complete before its CTAs exit (no PQKV_DEVERR_DRAIN) and leaves the
    context usable; the next call with the normal limit matches the oracle.
    Nothing is dropped or corrupted to cause the timeout: only the limit is
    short."""
    lens, qlens = [1500, 700, 300], [512, 200, 300]
    g, o, bt, cu, q = _build(case, lens, qlens, seed=77)
    seen = 0
    pq.set_decode_wait_limit_ns(1)
    try:
        for _ in range(5):
            _, e = _run(g, q, cu, bt, lens, 0.088)  # synchronized: no fault, no hang
            assert e & pq.DEVERR_DRAIN == 0, "work was still in flight when its CTA gave up draining"
            assert e & ~pq.DEVERR_TIMEOUT == 0
            seen += (e & pq.DEVERR_TIMEOUT) != 0
            if seen:
                break
    finally:
        pq.set_decode_wait_limit_ns(0)
    assert seen, "no wait ran out with a 1 ns limit"
    out, e = _run(g, q, cu, bt, lens, 0.088)
    assert e == 0
    ref, rerr = oracle.paged_prefill(o, q, cu, bt, np.array(lens, np.int32), 0.088)
    assert rerr == 0
    gh.assert_close(out, ref, case[0], tag="prefill after a timeout")
