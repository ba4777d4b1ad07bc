"""Block pool (host C++): allocation order, all-or-nothing semantics, sharing
with reference counts, and a random operation sequence checked against a
plain Python model of the same rules."""
import numpy as np
import pytest

pq = pytest.importorskip("paged_quantized_kv_cache_b200")


def test_fresh_pool_hands_out_lowest_ids_then_lifo():
    p = pq.BlockPool(10)
    assert p.num_free == 10
    assert list(p.alloc(3)) == [0, 1, 2]
    p.free([1])
    assert list(p.alloc(2)) == [1, 3]
    assert p.num_free == 6


def test_exhaustion_is_all_or_nothing():
    p = pq.BlockPool(5)
    p.alloc(4)
    with pytest.raises(pq.PqkvError) as e:
        p.alloc(2)
    assert e.value.status == pq.ERR_OOM
    assert p.num_free == 1
    assert list(p.alloc(1)) == [4]
    with pytest.raises(pq.PqkvError):
        p.alloc(1)


def test_sharing_and_refcounts():
    p = pq.BlockPool(4)
    ids = p.alloc(2)
    p.share(ids)
    p.share(ids[:1])
    assert [p.refcount(int(i)) for i in ids] == [3, 2]
    p.free(ids)
    assert p.num_free == 2
    p.free(ids)
    assert p.num_free == 3 and p.refcount(int(ids[1])) == 0
    p.free(ids[:1])
    assert p.num_free == 4


def test_state_errors_leave_the_pool_unchanged():
    p = pq.BlockPool(6)
    ids = p.alloc(3)
    with pytest.raises(pq.PqkvError) as e:
        p.free([ids[0], ids[0]])   # one reference, dropped twice
    assert e.value.status == pq.ERR_STATE
    assert p.refcount(int(ids[0])) == 1 and p.num_free == 3
    with pytest.raises(pq.PqkvError) as e:
        p.share([ids[1], 5])       # 5 is free
    assert e.value.status == pq.ERR_STATE
    assert p.refcount(int(ids[1])) == 1
    with pytest.raises(pq.PqkvError) as e:
        p.free([ids[2], 99])
    assert e.value.status == pq.ERR_ARG
    assert p.refcount(int(ids[2])) == 1
    assert p.refcount(99) == -1
    with pytest.raises(pq.PqkvError):
        pq.BlockPool(0)


def test_repeated_ids_in_one_free_return_a_block_once():
    p = pq.BlockPool(3)
    ids = p.alloc(1)
    p.share(ids)
    p.free([ids[0], ids[0]])
    assert p.num_free == 3
    got = set(int(x) for x in p.alloc(3))
    assert got == {0, 1, 2}


def test_random_operations_against_a_python_model():
    rng = np.random.default_rng(0)
    n = 200
    p = pq.BlockPool(n)
    refs = [0] * n
    free = list(range(n - 1, -1, -1))
    live = []
    for step in range(5000):
        op = rng.integers(0, 3)
        if op == 0:
            k = int(rng.integers(0, 12))
            if k > len(free):
                with pytest.raises(pq.PqkvError):
                    p.alloc(k)
                continue
            got = list(p.alloc(k))
            want = [free.pop() for _ in range(k)]
            assert got == want
            for i in got:
                refs[i] = 1
                live.append(i)
        elif op == 1 and live:
            ids = [live[int(j)] for j in rng.integers(0, len(live), size=int(rng.integers(1, 4)))]
            p.share(ids)
            for i in ids:
                refs[i] += 1
                live.append(i)
        elif op == 2 and live:
            picks = sorted(set(int(j) for j in rng.integers(0, len(live), size=int(rng.integers(1, 5)))),
                           reverse=True)
            ids = [live.pop(j) for j in picks]
            p.free(ids)
            returned = []
            for i in ids:
                refs[i] -= 1
            for i in ids:
                if refs[i] == 0 and i not in returned:
                    returned.append(i)
            free.extend(returned)
        assert p.num_free == len(free)
    assert all(p.refcount(i) == refs[i] for i in range(n))
