"""The C-ABI library loads and exports every entry point include/pqkv.h
declares; host-side logic (argument validation, cache sizes, slot mapping)
without a GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pqkv.h")

pq = pytest.importorskip("paged_quantized_kv_cache_b200")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pqkv_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = pq.lib()
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", pq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (pqkv_\w+)", out))
    assert set(names) == exported
    assert set(pq.EXPORTS) == set(names)


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "pqkv.h"\nint main(void){pqkv_pool* p = 0; (void)p; return PQKV_OK;}\n')
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-c",
                        str(src), "-o", str(tmp_path / "t.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_cache_layout_sizes():
    assert pq.cache_layout(pq.BF16, 10, 8, 128) == (10 * 8 * 2 * 16 * 256, 0, 0, 0)
    assert pq.cache_layout(pq.FP8_E4M3, 10, 8, 128) == (10 * 8 * 2 * 16 * 128, 10 * 8 * 16, 0, 0)
    assert pq.cache_layout(pq.FP4_E2M1, 10, 8, 128) == (10 * 8 * 2 * 16 * 64, 10 * 8 * 2 * 16 * 8,
                                                        10 * 8 * 2 * 8, 10 * 8 * 2 * 16 * 4 * 2)
    assert pq.cache_layout(pq.FP4_E2M1, 1, 1, 64)[1] == 2 * 16 * 4
    for bad in [(7, 1, 1, 64), (pq.BF16, 0, 1, 64), (pq.BF16, 1, 0, 64), (pq.BF16, 1, 1, 96)]:
        with pytest.raises(pq.PqkvError):
            pq.cache_layout(*bad)


def test_layout_matches_the_oracle_layout():
    import oracle
    for dt in range(5):
        for D in (64, 128):
            assert pq.cache_layout(dt, 3, 2, D) == oracle.cache_sizes(dt, 3, 2, D)


def test_invalid_arguments_are_rejected_before_any_launch():
    lib = pq.lib()
    null = None
    # bad dtype / head_dim / mismatched 16-bit dtypes / null pointers
    assert lib.pqkv_kv_cache_write(null, null, pq.BF16, 4, null, null, null, null, null, 9, 4, 1, 128,
                                   null, null) == pq.ERR_ARG
    assert lib.pqkv_kv_cache_write(null, null, pq.BF16, 4, null, null, null, null, null, pq.BF16, 4, 1, 96,
                                   null, null) == pq.ERR_ARG
    assert lib.pqkv_kv_cache_write(null, null, pq.FP16, 4, null, null, null, null, null, pq.BF16, 4, 1, 128,
                                   null, null) == pq.ERR_ARG
    assert lib.pqkv_kv_cache_write(null, null, pq.BF16, 4, null, null, null, null, null, pq.BF16, 4, 1, 128,
                                   null, null) == pq.ERR_ARG
    assert lib.pqkv_kv_cache_write(null, null, pq.BF16, 0, null, null, null, null, null, pq.BF16, 4, 1, 128,
                                   null, null) == pq.OK
    f = ctypes.c_float(0.1)
    # Hq not a multiple of Hkv, G > 8, batch beyond the limit, null buffers
    for (B, Hq, Hkv) in [(2, 6, 4), (2, 32, 2), (pq.MAX_BATCH + 1, 8, 8), (2, 8, 8)]:
        assert lib.pqkv_paged_decode_attention(null, pq.BF16, B, Hq, null, null, null, null, pq.BF16, 4, Hkv,
                                               128, null, 4, null, f, 0, null, null, 0, null,
                                               null) == pq.ERR_ARG
        # the entry point without a workspace checks the same sizes first
        assert lib.pqkv_paged_decode_attention_noalloc(null, pq.BF16, B, Hq, null, null, null, null, pq.BF16, 4,
                                                       Hkv, 128, null, 4, null, f, 0, null, null,
                                                       null) == pq.ERR_ARG
    # 12 query heads per KV head (a workspace size exists for 16 columns, but a
    # single-query decode takes at most 8): an argument error, not a scratch one
    assert lib.pqkv_paged_decode_attention_noalloc(null, pq.BF16, 2, 96, null, null, null, null, pq.BF16, 4, 8,
                                                   128, null, 4, null, f, 0, null, null, null) == pq.ERR_ARG
    # no sequences: nothing to do, but only for arguments the call accepts
    assert lib.pqkv_paged_decode_attention_noalloc(null, pq.BF16, 0, 32, null, null, null, null, pq.BF16, 4, 8,
                                                   128, null, 4, null, f, 0, null, null, null) == pq.OK
    assert lib.pqkv_paged_decode_attention_noalloc(null, pq.BF16, 0, 32, null, null, null, null, 9, 4, 8,
                                                   128, null, 4, null, f, 0, null, null, null) == pq.ERR_ARG
    assert lib.pqkv_paged_decode_attention_noalloc(null, pq.BF16, 0, 32, null, null, null, null, pq.BF16, 4, 8,
                                                   96, null, 4, null, f, 0, null, null, null) == pq.ERR_ARG
    assert lib.pqkv_decode_workspace_init(null, 16, null) == pq.ERR_ARG
    # workspace sizes: 0 for sizes no call accepts (checked before any device query)
    # (batch, Hq, Hkv, D, max_blocks, split): Hq not a multiple of Hkv, 32 columns
    # per KV head (at most 16 per pass), head_dim 96, no blocks, negative split, no batch
    for args in [(2, 6, 4, 128, 8, 0), (2, 64, 2, 128, 8, 0), (2, 8, 8, 96, 8, 0), (2, 8, 8, 128, 0, 0),
                 (2, 8, 8, 128, 8, -1), (0, 8, 8, 128, 8, 0)]:
        assert lib.pqkv_decode_workspace_bytes(*args) == 0
    # multi-query: q_len outside 1..64 or more than 8 query heads per KV head
    for (k, Hq, Hkv) in [(0, 32, 8), (65, 32, 8), (4, 48, 4), (4, 6, 4)]:
        assert lib.pqkv_multi_query_decode_workspace_bytes(2, k, Hq, Hkv, 128, 8, 0) == 0
        assert lib.pqkv_paged_multi_query_decode_attention(null, pq.BF16, 2, k, Hq, null, null, null, null, pq.BF16,
                                                           4, Hkv, 128, null, 4, null, f, 0, null, null, 0, null,
                                                           null) == pq.ERR_ARG
    assert lib.pqkv_encode(null, 5, pq.FP8_E4M3, null, null) == pq.ERR_ARG
    assert lib.pqkv_encode(null, 0, pq.BF16, null, null) == pq.ERR_ARG
    for s in range(6):
        assert lib.pqkv_status_string(s)


def test_build_slot_mapping():
    bt = np.array([[7, 3, -1], [2, -1, -1]], np.int32)
    s = pq.build_slot_mapping(bt, [14, 0], [4, 2])
    assert list(s) == [7 * 16 + 14, 7 * 16 + 15, 3 * 16 + 0, 3 * 16 + 1, 32, 33]
    with pytest.raises(pq.PqkvError):
        pq.build_slot_mapping(bt, [30, 0], [4, 1])   # needs table entry 2 (-1)
    with pytest.raises(pq.PqkvError):
        pq.build_slot_mapping(bt, [0, 0], [1, 17])   # second row's block 1 is -1
    assert pq.build_slot_mapping(bt, [5, 3], [0, 0]).size == 0


def test_slot_mapping_agrees_with_the_generator_formula():
    import workloads
    rng = np.random.default_rng(3)
    bt = rng.permutation(1000)[:60].reshape(3, 20).astype(np.int32)
    starts, news = [5, 100, 0], [40, 120, 320]
    got = pq.build_slot_mapping(bt, starts, news)
    want = np.concatenate([workloads.slots_for(bt[b], starts[b], news[b]) for b in range(3)])
    np.testing.assert_array_equal(got, want)
