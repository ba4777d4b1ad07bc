"""GPU parity of the whole-block moves against the oracle ("vLLM" glossary:
"PagedAttention" block sharing with copy-on-write for beam search / parallel
sampling; "Prefix caching"; "Preemption support": blocks swapped to CPU RAM).

Copies, swap records and swapped-in blocks must match the oracle bit for bit
(untouched blocks keep their poison); forked and prefix-shared sequences decode
to the oracle's outputs within the attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_helpers as gh
from tests.helpers import random_tables, slots

pytestmark = pytest.mark.gpu

pq = pytest.importorskip("paged_quantized_kv_cache_b200")

FORMATS = [(pq.FP16, 64, 2), (pq.BF16, 128, 8), (pq.FP8_E4M3, 128, 4), (pq.FP8_E5M2, 64, 1),
           (pq.FP4_E2M1, 128, 8), (pq.FP4_E2M1, 64, 3)]


def _filled(kv_dtype, D, H, nb, seed, lens=(70, 33, 16, 5)):
    rng = np.random.default_rng(seed)
    bt = random_tables(rng, list(lens), nb)
    g, o = gh.new_pair(kv_dtype, nb, H, D)
    dt = torch.float16 if kv_dtype == pq.FP16 else torch.bfloat16
    for b, L in enumerate(lens):
        k = rng.standard_normal((L, H, D)).astype(np.float32)
        v = rng.standard_normal((L, H, D)).astype(np.float32)
        k[:, :, 3] *= 16
        kt, vt = torch.from_numpy(k).to(dt), torch.from_numpy(v).to(dt)
        ge, oe = gh.write_both(g, o, kt, vt, slots(bt[b], 0, L))
        assert ge == oe == 0
    return rng, bt, g, o


@pytest.mark.parametrize("kv_dtype,D,H", FORMATS)
def test_copy_blocks_bit_exact(kv_dtype, D, H):
    nb = 48
    rng, bt, g, o = _filled(kv_dtype, D, H, nb, seed=10 + kv_dtype)
    used = sorted(set(int(x) for x in bt.ravel() if x >= 0))
    spare = [i for i in range(nb) if i not in set(used)]
    src = rng.choice(used, size=6, replace=False)
    dst = rng.choice(spare, size=6, replace=False)
    pairs = np.stack([src, dst], axis=1).astype(np.int32)
    pairs = np.concatenate([pairs, [[0, nb]], [[-1, int(spare[0])]]]).astype(np.int32)
    e = gh.err_flag()
    pq.copy_blocks(g, torch.from_numpy(pairs).cuda(), e)
    oe = oracle.copy_blocks(o, pairs)
    torch.cuda.synchronize()
    assert int(e.item()) == oe == pq.DEVERR_BLOCK_ID
    gh.assert_cache_equal(g, o, tag="copy")


@pytest.mark.parametrize("kv_dtype,D,H", FORMATS)
def test_swap_out_and_in_bit_exact(kv_dtype, D, H):
    nb = 40
    rng, bt, g, o = _filled(kv_dtype, D, H, nb, seed=20 + kv_dtype)
    ids = bt[0][bt[0] >= 0].astype(np.int32)
    rec = pq.block_record_bytes(kv_dtype, H, D)
    assert rec == oracle.block_record_bytes(kv_dtype, H, D)
    host = torch.empty(ids.size * rec, dtype=torch.uint8).pin_memory()
    host.fill_(0xAB)
    e = gh.err_flag()
    pq.swap_out(g, torch.from_numpy(ids).cuda(), host, e)
    torch.cuda.synchronize()
    want = np.zeros((ids.size, rec), dtype=np.uint8)
    assert oracle.swap_out(o, ids, want) == 0 and int(e.item()) == 0
    np.testing.assert_array_equal(host.numpy().reshape(ids.size, rec), want)
    used = set(int(x) for x in bt.ravel() if x >= 0)
    back = np.array([i for i in range(nb) if i not in used][:ids.size], dtype=np.int32)
    back_err = np.concatenate([back, [nb]]).astype(np.int32)
    host2 = torch.empty((ids.size + 1) * rec, dtype=torch.uint8).pin_memory()
    host2[:ids.size * rec].copy_(host)
    pq.swap_in(g, torch.from_numpy(back_err).cuda(), host2, e)
    oe = oracle.swap_in(o, back_err, np.concatenate([want, np.zeros((1, rec), np.uint8)]))
    torch.cuda.synchronize()
    assert int(e.item()) == oe == pq.DEVERR_BLOCK_ID
    gh.assert_cache_equal(g, o, tag="swap")


def test_swap_rejects_pageable_host_memory():
    g = pq.allocate_cache(pq.BF16, 4, 1, 64)
    with pytest.raises(ValueError):
        pq.swap_out(g, torch.zeros(1, dtype=torch.int32, device="cuda"), torch.empty(64 * 64, dtype=torch.uint8),
                    gh.err_flag())


@pytest.mark.parametrize("kv_dtype,qdt", [(pq.BF16, torch.bfloat16), (pq.FP8_E4M3, torch.bfloat16),
                                          (pq.FP4_E2M1, torch.float16)])
def test_fork_with_copy_on_write_then_append(kv_dtype, qdt):
    """Parallel sampling: sequence B forks off A (sharing every block, the last one
    partial); each then appends its own tokens. B's write into the shared partial
    block goes through pool.cow + copy_blocks; both decode like the oracle doing
    the same steps, and A's cache is untouched by B."""
    rng = np.random.default_rng(30)
    H, Hq, D, nb = 4, 16, 128, 32
    pool = pq.BlockPool(nb)
    L0 = 53
    ida = pool.alloc((L0 + 15) // 16)
    g, o = gh.new_pair(kv_dtype, nb, H, D)
    k = torch.from_numpy(rng.standard_normal((L0 + 9, H, D)).astype(np.float32)).to(qdt)
    v = torch.from_numpy(rng.standard_normal((L0 + 9, H, D)).astype(np.float32)).to(qdt)
    ge, oe = gh.write_both(g, o, k[:L0], v[:L0], slots(ida, 0, L0))
    assert ge == oe == 0
    pool.share(ida)  # B = fork of A
    idb = ida.copy()
    last = int(idb[-1])
    new, need = pool.cow(last)
    assert need
    idb[-1] = new
    pairs = np.array([[last, new]], dtype=np.int32)
    e = gh.err_flag()
    pq.copy_blocks(g, torch.from_numpy(pairs).cuda(), e)
    assert oracle.copy_blocks(o, pairs) == 0
    # each appends 5 different tokens (A: rows L0.., B: rows L0+4..)
    ga, oa = gh.write_both(g, o, k[L0:L0 + 5], v[L0:L0 + 5], slots(ida, L0, 5))
    gb, ob = gh.write_both(g, o, k[L0 + 4:L0 + 9], v[L0 + 4:L0 + 9], slots(idb, L0, 5))
    assert ga == oa == gb == ob == 0 and int(e.item()) == 0
    gh.assert_cache_equal(g, o, tag="fork")
    tables = np.stack([ida, idb]).astype(np.int32)
    lens = np.array([L0 + 5, L0 + 5], dtype=np.int32)
    q = torch.from_numpy(rng.standard_normal((2, Hq, D)).astype(np.float32)).to(qdt)
    q[1] = q[0]
    scale = 1.0 / np.sqrt(D)
    out, err = gh.decode_gpu(g, q, tables, lens, scale)
    ref, rerr = oracle.paged_decode(o, q, tables, lens, scale)
    assert err == rerr == 0
    gh.assert_close(out, ref, kv_dtype, tag="fork")
    # the two sequences differ only in their last 5 tokens
    assert not torch.equal(out[0], out[1])


def test_prefix_cache_reuse_decodes_like_a_private_copy():
    """Request 2 shares request 1's cached prompt blocks (prefix lookup) and
    writes only its own tail; decoding it equals decoding a private layout of
    the same tokens, bit for bit."""
    rng = np.random.default_rng(31)
    H, Hq, D, nb = 8, 32, 128, 64
    pool = pq.BlockPool(nb)
    prompt = rng.integers(0, 32000, size=200).astype(np.int32)
    kv_of = {}

    def kv_for(tok):  # the same token at the same position gives the same K/V
        key = int(tok)
        if key not in kv_of:
            r = np.random.default_rng(key)
            kv_of[key] = (r.standard_normal((H, D)).astype(np.float32), r.standard_normal((H, D)).astype(np.float32))
        return kv_of[key]

    def write_tokens(g, ids, toks, start):
        k = torch.from_numpy(np.stack([kv_for(t)[0] for t in toks])).to(torch.bfloat16)
        v = torch.from_numpy(np.stack([kv_for(t)[1] for t in toks])).to(torch.bfloat16)
        e = gh.err_flag()
        pq.kv_cache_write(k.cuda(), v.cuda(), torch.from_numpy(slots(ids, start, len(toks))).cuda(), g, e)
        torch.cuda.synchronize()
        assert int(e.item()) == 0

    g = pq.allocate_cache(pq.BF16, nb, H, D, fill=0xFF)
    ids1 = pool.alloc((prompt.size + 15) // 16)
    write_tokens(g, ids1, prompt, 0)
    pool.prefix_insert(prompt, ids1)
    second = np.concatenate([prompt[:176], rng.integers(0, 32000, size=30).astype(np.int32)])
    hit = pool.prefix_lookup(second)
    assert hit.size == 11 and list(hit) == list(ids1[:11])
    tail = pool.alloc((second.size + 15) // 16 - hit.size)
    ids2 = np.concatenate([hit, tail]).astype(np.int32)
    write_tokens(g, ids2, second[176:], 176)
    private = pool.alloc((second.size + 15) // 16)
    write_tokens(g, private, second, 0)
    q = torch.from_numpy(rng.standard_normal((1, Hq, D)).astype(np.float32)).to(torch.bfloat16)
    lens = np.array([second.size], dtype=np.int32)
    a, ea = gh.decode_gpu(g, q, ids2[None], lens, 0.088)
    b, eb = gh.decode_gpu(g, q, private[None], lens, 0.088)
    assert ea == eb == 0
    assert torch.equal(a, b)
