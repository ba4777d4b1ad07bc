"""Prefix cache and copy-on-write of the host block pool ("vLLM" glossary:
"Prefix caching", "Automatic prefix caching", "PagedAttention" block sharing
for beam search / parallel sampling), and the oracle's whole-block moves
("PagedAttention" copy for a forked shared block; "Preemption support":
blocks swapped to CPU RAM and back), pinned through the oracle's gather."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import random_tables, slots

pq = pytest.importorskip("paged_quantized_kv_cache_b200")

BS = 16


def _prompt(rng, n):
    return rng.integers(0, 50000, size=n).astype(np.int32)


def test_same_prompt_hits_all_full_blocks():
    rng = np.random.default_rng(0)
    p = pq.BlockPool(32)
    toks = _prompt(rng, 5 * BS + 7)
    ids = p.alloc(6)
    p.prefix_insert(toks, ids)
    assert p.num_cached == 5  # the partial sixth block is never cached
    hit = p.prefix_lookup(toks)
    assert list(hit) == list(ids[:5])
    assert [p.refcount(int(i)) for i in ids] == [2] * 5 + [1]


def test_common_prefix_hits_exactly_the_shared_blocks():
    rng = np.random.default_rng(1)
    p = pq.BlockPool(64)
    a = _prompt(rng, 8 * BS)
    ids = p.alloc(8)
    p.prefix_insert(a, ids)
    for k in range(0, 8):
        b = a.copy()
        b[k * BS + 3] += 1  # first difference inside block k
        assert list(p.prefix_lookup(b)) == list(ids[:k])
    # a block's identity includes everything before it: block 1 of `a` after
    # a different block 0 is a miss
    c = a.copy()
    c[:BS] = _prompt(rng, BS)
    assert p.prefix_lookup(c).size == 0


def test_lookup_of_a_shorter_prompt_and_token_granularity():
    rng = np.random.default_rng(2)
    p = pq.BlockPool(16)
    a = _prompt(rng, 4 * BS)
    ids = p.alloc(4)
    p.prefix_insert(a, ids)
    assert list(p.prefix_lookup(a[:3 * BS + 15])) == list(ids[:3])
    assert p.prefix_lookup(a[:BS - 1]).size == 0


def test_released_cached_blocks_are_evictable_and_revived_by_lookup():
    rng = np.random.default_rng(3)
    p = pq.BlockPool(8)
    a = _prompt(rng, 3 * BS)
    ids = p.alloc(3)
    p.prefix_insert(a, ids)
    p.free(ids)
    assert p.num_free == 5 and p.num_evictable == 3 and p.num_cached == 3
    hit = p.prefix_lookup(a)
    assert list(hit) == list(ids)
    assert p.num_evictable == 0 and all(p.refcount(int(i)) == 1 for i in ids)


def test_alloc_takes_free_blocks_first_then_evicts_least_recently_released():
    rng = np.random.default_rng(4)
    p = pq.BlockPool(6)
    a, b = _prompt(rng, 2 * BS), _prompt(rng, 2 * BS)
    ia = p.alloc(2)
    p.prefix_insert(a, ia)
    ib = p.alloc(2)
    p.prefix_insert(b, ib)
    p.free(ia[::-1])  # released: ia[1] then ia[0]
    p.free(ib)
    got = p.alloc(2)  # the two never-used blocks
    assert set(got) == {4, 5} and p.num_evictable == 4
    got = p.alloc(1)  # least recently released: ia[1]
    assert list(got) == [ia[1]] and p.num_cached == 3
    # a's first block is still cached, its second is gone
    assert list(p.prefix_lookup(a)) == [ia[0]]
    with pytest.raises(pq.PqkvError) as e:
        p.alloc(4)  # 2 evictable (b) + 0 free < 4: no change
    assert e.value.status == pq.ERR_OOM and p.num_evictable == 2


def test_evicted_block_reused_for_other_tokens_cannot_revive_old_children():
    rng = np.random.default_rng(5)
    p = pq.BlockPool(3)
    a = _prompt(rng, 2 * BS)
    ia = p.alloc(2)
    p.prefix_insert(a, ia)
    p.free([ia[0]])          # first block evictable, second still referenced
    other = p.alloc(2)       # 1 free + evicts ia[0]
    assert ia[0] in other
    c = _prompt(rng, BS)
    p.prefix_insert(c, [ia[0]])  # the same id now caches other tokens
    # c followed by a's second block must not hit a's second block
    probe = np.concatenate([c, a[BS:]])
    assert list(p.prefix_lookup(probe)) == [ia[0]]
    # and a itself misses entirely (its first block was evicted)
    assert p.prefix_lookup(a).size == 0


def test_insert_checks_before_changing_anything():
    rng = np.random.default_rng(6)
    p = pq.BlockPool(8)
    a, b = _prompt(rng, 2 * BS), _prompt(rng, 2 * BS)
    ia = p.alloc(2)
    p.prefix_insert(a, ia)
    ib = p.alloc(1)
    with pytest.raises(pq.PqkvError) as e:
        p.prefix_insert(b, [ib[0], ia[1]])  # ia[1] is cached under a's prefix
    assert e.value.status == pq.ERR_STATE and p.num_cached == 2
    with pytest.raises(pq.PqkvError) as e:
        p.prefix_insert(b, [ib[0], ib[0]])  # repeated id
    assert e.value.status == pq.ERR_STATE and p.num_cached == 2
    free_id = p.alloc(1)[0]
    p.free([free_id])
    with pytest.raises(pq.PqkvError) as e:
        p.prefix_insert(b, [free_id])  # not referenced
    assert e.value.status == pq.ERR_STATE
    # re-inserting the same prompt with a duplicate computation keeps the first
    dup = p.alloc(2)
    p.prefix_insert(a, dup)
    assert list(p.prefix_lookup(a)) == list(ia) and p.num_cached == 2


def test_cow_only_copies_shared_or_cached_blocks():
    p = pq.BlockPool(6)
    (x,) = p.alloc(1)
    assert p.cow(int(x)) == (x, False)
    p.share([x])
    new, need = p.cow(int(x))
    assert need and new != x and p.refcount(int(x)) == 1 and p.refcount(new) == 1
    toks = np.arange(BS, dtype=np.int32)
    p.prefix_insert(toks, [new])
    new2, need2 = p.cow(new)  # cached: writing it would corrupt the entry
    assert need2 and new2 != new and p.refcount(new) == 0 and p.num_evictable == 1
    with pytest.raises(pq.PqkvError) as e:
        p.cow(new)
    assert e.value.status == pq.ERR_STATE


def test_random_prefix_operations_keep_the_books_balanced():
    """Every id is exactly one of: referenced, evictable, free."""
    rng = np.random.default_rng(7)
    nb = 40
    p = pq.BlockPool(nb)
    base = _prompt(rng, 6 * BS)
    live = []
    for step in range(400):
        op = rng.integers(0, 3)
        if op == 0:
            n = int(rng.integers(1, 7)) * BS
            toks = base[:n].copy()
            if rng.random() < 0.5:
                toks[int(rng.integers(0, n))] += 1
            hit = p.prefix_lookup(toks)
            need = n // BS - hit.size
            try:
                new = p.alloc(need)
            except pq.PqkvError:
                p.free(hit)
                continue
            ids = np.concatenate([hit, new]).astype(np.int32)
            p.prefix_insert(toks, ids)
            live.append(ids)
        elif op == 1 and live:
            p.free(live.pop(int(rng.integers(0, len(live)))))
        elif op == 2 and live:
            ids = live[int(rng.integers(0, len(live)))]
            j = int(rng.integers(0, ids.size))
            try:
                ids[j], _ = p.cow(int(ids[j]))
            except pq.PqkvError as e:
                assert e.status == pq.ERR_OOM
        refs = sum(1 for i in range(nb) if p.refcount(i) > 0)
        assert refs + p.num_evictable + p.num_free == nb
    for ids in live:
        p.free(ids)
    assert p.num_free + p.num_evictable == nb


@pytest.mark.parametrize("dt", [oracle.DT_BF16, oracle.DT_E4M3, oracle.DT_E2M1])
def test_oracle_block_copy_and_swap_round_trip(dt):
    rng = np.random.default_rng(8)
    H, D, nb = 2, 64, 12
    lens = [40, 21]
    bt = random_tables(rng, lens, nb)
    c = oracle.Cache(dt, nb, H, D)
    for b, L in enumerate(lens):
        k = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(torch.bfloat16)
        v = torch.from_numpy(rng.standard_normal((L, H, D), dtype=np.float32)).to(torch.bfloat16)
        oracle.kv_cache_write(c, k, v, slots(bt[b], 0, L))
    used = set(int(x) for x in bt.ravel() if x >= 0)
    spare = [i for i in range(nb) if i not in used]
    # copy-on-write: a forked table pointing at copies reads back the same K/V
    row = bt[0].copy()
    pairs = [(int(row[j]), spare[j]) for j in range(3)]
    assert oracle.copy_blocks(c, pairs) == 0
    fork = row.copy()
    fork[:3] = spare[:3]
    for h in range(H):
        a = oracle.gather(c, row, lens[0], h)
        f = oracle.gather(c, fork, lens[0], h)
        for x, y in zip(a, f):
            np.testing.assert_array_equal(x, y)
    # swap out sequence 1's blocks, back into other ids
    rec = oracle.block_record_bytes(dt, H, D)
    assert rec == sum(x.size // nb for x in c.arrays() if x is not None)
    ids = bt[1][bt[1] >= 0]
    records = np.zeros((ids.size, rec), dtype=np.uint8)
    assert oracle.swap_out(c, ids, records) == 0
    back = np.array(spare[3:3 + ids.size], dtype=np.int32)
    assert oracle.swap_in(c, back, records) == 0
    moved = bt[1].copy()
    moved[:ids.size] = back
    for h in range(H):
        a = oracle.gather(c, bt[1], lens[1], h)
        f = oracle.gather(c, moved, lens[1], h)
        for x, y in zip(a, f):
            np.testing.assert_array_equal(x, y)
    assert oracle.copy_blocks(c, [(0, nb)]) == oracle.ERR_BLOCK_ID
    assert oracle.swap_out(c, [-1], records[:1]) == oracle.ERR_BLOCK_ID
