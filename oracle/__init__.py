"""CPU oracle for the paged, quantized KV cache -- TEST INFRASTRUCTURE ONLY.

A ctypes wrapper around pqkv_oracle.c (plain C, fp64 attention). Only the test
suite, the package smoke check and the benchmark's CPU-baseline leg may import
this package. It shares no code with the GPU library and never imports it.

Page citations (by title and section) are in pqkv_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pqkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib: Optional[ctypes.CDLL] = None

DT_FP16, DT_BF16, DT_E4M3, DT_E5M2, DT_E2M1 = 0, 1, 2, 3, 4
ERR_SLOT, ERR_BLOCK_ID, ERR_SEQ_LEN, ERR_RUN = 1, 2, 4, 8
BLOCK = 16


def build(force: bool = False) -> str:
    """Compile pqkv_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", "-Wall", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_encode.argtypes = [I, P, ctypes.c_int64, P]
        _lib.oracle_encode_fp16.argtypes = [P, ctypes.c_int64, P]
        _lib.oracle_decode.argtypes = [I, P, ctypes.c_int64, P]
        _lib.oracle_decode_fp16.argtypes = [P, ctypes.c_int64, P]
        _lib.oracle_kv_cache_write.argtypes = [P, P, I, I, P, P, P, P, P, I, I, I, I, P]
        _lib.oracle_kv_cache_write.restype = I
        _lib.oracle_gather.argtypes = [P, P, P, P, I, I, I, I, P, I, I, P, P, P]
        _lib.oracle_paged_decode.argtypes = [P, I, ctypes.c_int, I, P, P, P, P, I, I, I, I, P, I, P,
                                             ctypes.c_float, P, P]
        _lib.oracle_paged_decode.restype = I
        _lib.oracle_paged_prefill.argtypes = [P, I, P, I, I, P, P, P, P, I, I, I, I, P, I, P,
                                              ctypes.c_float, P, P]
        _lib.oracle_paged_prefill.restype = I
        _lib.oracle_num_threads.restype = I
    return _lib


def _ptr(a) -> Optional[int]:
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        assert a.is_contiguous() and a.device.type == "cpu"
        return a.data_ptr()
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ---- number formats -------------------------------------------------------

def encode(dt: int, x: np.ndarray) -> np.ndarray:
    """float32 -> codes of FP8 E4M3 / E5M2 / E2M1 (nearest even, satfinite)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_encode(dt, _ptr(x), x.size, _ptr(out))
    return out


def encode_fp16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_encode_fp16(_ptr(x), x.size, _ptr(out))
    return out


def decode(dt: int, codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    lib().oracle_decode(dt, _ptr(codes), codes.size, _ptr(out))
    return out


def decode_fp16(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint16)
    out = np.empty(codes.shape, dtype=np.float64)
    lib().oracle_decode_fp16(_ptr(codes), codes.size, _ptr(out))
    return out


# ---- cache ----------------------------------------------------------------

def cache_sizes(dt: int, nb: int, H: int, D: int) -> Tuple[int, int, int, int]:
    """Bytes of (cache, scales, outliers_idx, outliers_val) in the oracle's layout."""
    if dt in (DT_FP16, DT_BF16):
        return nb * H * 2 * BLOCK * D * 2, 0, 0, 0
    if dt in (DT_E4M3, DT_E5M2):
        return nb * H * 2 * BLOCK * D, nb * H * 4 * 4, 0, 0
    return (nb * H * 2 * BLOCK * D // 2, nb * H * 2 * BLOCK * (D // 16),
            nb * H * 2 * 8, nb * H * 2 * BLOCK * 4 * 2)


class Cache:
    """Host-side cache arrays (numpy uint8), filled with a poison byte pattern."""

    def __init__(self, dt: int, nb: int, H: int, D: int, poison: bool = True):
        self.dt, self.nb, self.H, self.D = dt, nb, H, D
        sizes = cache_sizes(dt, nb, H, D)
        fill = 0xFF if poison else 0
        self.cache = np.full(sizes[0], fill, dtype=np.uint8)
        self.scales = np.full(sizes[1], fill, dtype=np.uint8) if sizes[1] else None
        self.oidx = np.full(sizes[2], fill, dtype=np.uint8) if sizes[2] else None
        self.oval = np.full(sizes[3], fill, dtype=np.uint8) if sizes[3] else None

    def arrays(self):
        return self.cache, self.scales, self.oidx, self.oval


def _u16(x: torch.Tensor) -> torch.Tensor:
    return x.contiguous().view(torch.int16)


def kv_cache_write(c: Cache, k: torch.Tensor, v: torch.Tensor, slots: np.ndarray) -> int:
    """Apply one write call to the host cache. Returns the error bits."""
    in_dt = DT_BF16 if k.dtype == torch.bfloat16 else DT_FP16
    T = k.shape[0]
    assert k.shape == (T, c.H, c.D) and v.shape == k.shape
    slots = np.ascontiguousarray(slots, dtype=np.int32)
    err = np.zeros(1, dtype=np.int32)
    ku, vu = _u16(k), _u16(v)
    rc = lib().oracle_kv_cache_write(_ptr(ku), _ptr(vu), in_dt, T, _ptr(slots), _ptr(c.cache),
                                     _ptr(c.scales), _ptr(c.oidx), _ptr(c.oval), c.dt, c.nb, c.H,
                                     c.D, _ptr(err))
    if rc != 0:
        raise ValueError("oracle write rejected its arguments")
    return int(err[0])


def gather(c: Cache, table_row: np.ndarray, L: int, h: int):
    """Dequantized K, V [L][D] (fp64) of one sequence and KV head, and validity."""
    table_row = np.ascontiguousarray(table_row, dtype=np.int32)
    kd = np.zeros((L, c.D), dtype=np.float64)
    vd = np.zeros((L, c.D), dtype=np.float64)
    valid = np.zeros(L, dtype=np.uint8)
    lib().oracle_gather(_ptr(c.cache), _ptr(c.scales), _ptr(c.oidx), _ptr(c.oval), c.dt, c.nb,
                        c.H, c.D, _ptr(table_row), L, h, _ptr(kd), _ptr(vd), _ptr(valid))
    return kd, vd, valid.astype(bool)


def paged_decode(c: Cache, q: torch.Tensor, block_tables: np.ndarray, seq_lens: np.ndarray,
                 scale: float) -> Tuple[np.ndarray, int]:
    """fp64 attention output [B][Hq][D] and the error bits."""
    B, Hq, D = q.shape
    assert D == c.D
    q_dt = DT_BF16 if q.dtype == torch.bfloat16 else DT_FP16
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    err = np.zeros(1, dtype=np.int32)
    qu = _u16(q)
    rc = lib().oracle_paged_decode(_ptr(qu), q_dt, B, Hq, _ptr(c.cache), _ptr(c.scales),
                                   _ptr(c.oidx), _ptr(c.oval), c.dt, c.nb, c.H, c.D, _ptr(bt),
                                   bt.shape[1], _ptr(sl), ctypes.c_float(scale), _ptr(out),
                                   _ptr(err))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return out, int(err[0])


def paged_prefill(c: Cache, q: torch.Tensor, cu_q: np.ndarray, block_tables: np.ndarray,
                  seq_lens: np.ndarray, scale: float) -> Tuple[np.ndarray, int]:
    """Causal chunked-prefill attention: q [cu_q[-1]][Hq][D]; sequence b's query
    tokens are its last cu_q[b+1] - cu_q[b] positions. fp64 output, error bits."""
    T, Hq, D = q.shape
    assert D == c.D
    q_dt = DT_BF16 if q.dtype == torch.bfloat16 else DT_FP16
    cu = np.ascontiguousarray(cu_q, dtype=np.int32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B = sl.size
    assert cu.size == B + 1 and cu[-1] == T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    err = np.zeros(1, dtype=np.int32)
    qu = _u16(q)
    rc = lib().oracle_paged_prefill(_ptr(qu), q_dt, _ptr(cu), B, Hq, _ptr(c.cache), _ptr(c.scales),
                                    _ptr(c.oidx), _ptr(c.oval), c.dt, c.nb, c.H, c.D, _ptr(bt),
                                    bt.shape[1], _ptr(sl), ctypes.c_float(scale), _ptr(out), _ptr(err))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments")
    return out, int(err[0])


# ---- whole-block moves ------------------------------------------------------
# "vLLM" glossary, "PagedAttention": blocks shared across sequences (beam search,
# parallel sampling), so a sequence writing into a shared block takes its own
# copy first; "Preemption support": KV cache blocks swapped out to CPU RAM and
# back. A block is the same slice of each cache array (all arrays are
# [num_blocks][...]); its record is those slices in array order: codes, scales,
# outlier indices, outlier values.

def _block_views(c: Cache):
    return [a.reshape(c.nb, -1) for a in c.arrays() if a is not None]


def block_record_bytes(dt: int, H: int, D: int) -> int:
    return sum(cache_sizes(dt, 1, H, D))


def copy_blocks(c: Cache, pairs) -> int:
    """Copy block src into block dst for each (src, dst), in order. Returns error bits."""
    err = 0
    for s, d in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        if not (0 <= s < c.nb and 0 <= d < c.nb):
            err |= ERR_BLOCK_ID
            continue
        for v in _block_views(c):
            v[d] = v[s]
    return err


def swap_out(c: Cache, ids, records: np.ndarray) -> int:
    """Record i = block ids[i]'s slices, concatenated. records: uint8 [n][record bytes]."""
    err = 0
    for i, b in enumerate(np.asarray(ids, dtype=np.int64).ravel()):
        if not (0 <= b < c.nb):
            err |= ERR_BLOCK_ID
            continue
        records[i] = np.concatenate([v[b] for v in _block_views(c)])
    return err


def swap_in(c: Cache, ids, records: np.ndarray) -> int:
    """Inverse of swap_out: record i back into block ids[i]."""
    err = 0
    for i, b in enumerate(np.asarray(ids, dtype=np.int64).ravel()):
        if not (0 <= b < c.nb):
            err |= ERR_BLOCK_ID
            continue
        off = 0
        for v in _block_views(c):
            v[b] = records[i, off:off + v.shape[1]]
            off += v.shape[1]
    return err
