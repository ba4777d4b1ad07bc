"""The read-bandwidth probe (pqkv_read_probe) reads exactly the K|V tiles a
decode of the same batch reads: its checksum (XOR of one word per tile, the
word at byte 16 * (flat index mod 8) of the tile) is recomputed here from the
cache bytes and the block tables, and a bad block id is flagged and skipped."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
pq = pytest.importorskip("paged_quantized_kv_cache_b200")

TILE_ROW = {pq.BF16: lambda D: 2 * D, pq.FP8_E4M3: lambda D: D, pq.FP4_E2M1: lambda D: D // 2}


def expected_checksum(cache_bytes, bt, lens, H, tile, nb):
    words = cache_bytes.view(np.uint32)
    x = 0
    f = 0
    for b, L in enumerate(lens):
        n = (int(L) + 15) // 16
        for h in range(H):
            for j in range(n):
                bid = int(bt[b, j])
                if 0 <= bid < nb:
                    off = ((bid * H + h) * tile + (f & 7) * 16) // 4
                    x ^= int(words[off])
                f += 1
    return x


@pytest.mark.parametrize("kv_dtype", [pq.BF16, pq.FP8_E4M3, pq.FP4_E2M1])
@pytest.mark.parametrize("D", [64, 128])
def test_read_probe_checksum(kv_dtype, D):
    rng = np.random.default_rng(11 + kv_dtype + D)
    H, nb = 3, 96
    lens = np.array([17, 0, 100, 33, 256, 1], np.int32)
    nblk = [(int(L) + 15) // 16 for L in lens]
    bt = np.full((len(lens), 20), -1, np.int32)
    ids = rng.permutation(nb)
    pos = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = ids[pos:pos + n]
        pos += n
    g = pq.allocate_cache(kv_dtype, nb, H, D)
    host = rng.integers(0, 256, g.cache.numel(), dtype=np.uint8)
    g.cache.copy_(torch.from_numpy(host))
    tile = 2 * 16 * TILE_ROW[kv_dtype](D)
    for bad in (False, True):
        t = bt.copy()
        if bad:
            t[2, 3] = nb + 5
        chk = torch.zeros(1, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pq.read_probe(g, torch.from_numpy(t).cuda(), torch.from_numpy(lens).cuda(), chk, err)
        torch.cuda.synchronize()
        assert int(err.item()) == (pq.DEVERR_BLOCK_ID if bad else 0)
        want = expected_checksum(host, t, lens, H, tile, nb)
        assert (int(chk.item()) & 0xFFFFFFFF) == want
