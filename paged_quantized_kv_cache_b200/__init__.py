"""Paged, quantized KV-cache decode attention for B200 -- Python binding.

Argument marshalling only: every step runs in libpqkv.so (CUDA kernels for
sm_100a and a C++ block pool) through its C ABI (include/pqkv.h). PyTorch is
used for device memory and streams. If the library is missing this module
raises at import; there is no other code path.

Build the library with ``python -m paged_quantized_kv_cache_b200.build``; the
first call into this module loads it and raises ImportError if it is missing.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpqkv.so")

FP16, BF16, FP8_E4M3, FP8_E5M2, FP4_E2M1 = 0, 1, 2, 3, 4
DTYPE_NAMES = {FP16: "fp16", BF16: "bf16", FP8_E4M3: "fp8_e4m3", FP8_E5M2: "fp8_e5m2", FP4_E2M1: "fp4_e2m1"}
OK, ERR_ARG, ERR_OOM, ERR_STATE, ERR_CUDA, ERR_SCRATCH = 0, 1, 2, 3, 4, 5
NOALLOC_SCRATCH_BYTES = 16 << 20
DEVERR_SLOT, DEVERR_BLOCK_ID, DEVERR_SEQ_LEN, DEVERR_RUN, DEVERR_TIMEOUT, DEVERR_DRAIN = 1, 2, 4, 8, 16, 32
BLOCK_SIZE = 16
MAX_BATCH = 4096

# Every C entry point the library exports (must match include/pqkv.h).
EXPORTS = (
    "pqkv_version", "pqkv_status_string", "pqkv_cache_layout", "pqkv_kv_cache_write",
    "pqkv_decode_workspace_bytes", "pqkv_paged_decode_attention", "pqkv_decode_workspace_init",
    "pqkv_encode", "pqkv_pool_create", "pqkv_pool_destroy", "pqkv_pool_alloc", "pqkv_pool_share",
    "pqkv_pool_free", "pqkv_pool_num_free", "pqkv_pool_refcount", "pqkv_build_slot_mapping",
    "pqkv_paged_decode_attention_noalloc", "pqkv_pool_num_evictable", "pqkv_pool_num_cached",
    "pqkv_pool_prefix_lookup", "pqkv_pool_prefix_insert", "pqkv_pool_cow", "pqkv_copy_blocks",
    "pqkv_block_record_bytes", "pqkv_swap_out", "pqkv_swap_in", "pqkv_paged_prefill_attention",
    "pqkv_paged_multi_query_decode_attention", "pqkv_multi_query_decode_workspace_bytes",
    "pqkv_read_probe", "pqkv_set_decode_wait_limit_ns",
)


class PqkvError(RuntimeError):
    def __init__(self, func: str, status: int):
        super().__init__("%s failed: %s (%d)" % (func, lib().pqkv_status_string(status).decode(), status))
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libpqkv.so is not built (run: python -m paged_quantized_kv_cache_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "pqkv_version": (I, []),
        "pqkv_status_string": (ctypes.c_char_p, [I]),
        "pqkv_cache_layout": (I, [I, I, I, I, P]),
        "pqkv_kv_cache_write": (I, [P, P, I, I, P, P, P, P, P, I, I, I, I, P, P]),
        "pqkv_decode_workspace_bytes": (Z, [I, I, I, I, I, I]),
        "pqkv_multi_query_decode_workspace_bytes": (Z, [I, I, I, I, I, I, I]),
        "pqkv_paged_decode_attention": (I, [P, I, I, I, P, P, P, P, I, I, I, I, P, I, P, ctypes.c_float, I,
                                            P, P, Z, P, P]),
        "pqkv_decode_workspace_init": (I, [P, Z, P]),
        "pqkv_encode": (I, [P, ctypes.c_int64, I, P, P]),
        "pqkv_pool_create": (I, [ctypes.c_int32, ctypes.POINTER(P)]),
        "pqkv_pool_destroy": (None, [P]),
        "pqkv_pool_alloc": (I, [P, I, P]),
        "pqkv_pool_share": (I, [P, P, I]),
        "pqkv_pool_free": (I, [P, P, I]),
        "pqkv_pool_num_free": (ctypes.c_int32, [P]),
        "pqkv_pool_refcount": (ctypes.c_int32, [P, ctypes.c_int32]),
        "pqkv_build_slot_mapping": (I, [P, I, I, P, P, P]),
        "pqkv_paged_decode_attention_noalloc": (I, [P, I, I, I, P, P, P, P, I, I, I, I, P, I, P, ctypes.c_float,
                                                    I, P, P, P]),
        "pqkv_pool_num_evictable": (ctypes.c_int32, [P]),
        "pqkv_pool_num_cached": (ctypes.c_int32, [P]),
        "pqkv_pool_prefix_lookup": (I, [P, P, I, P, ctypes.POINTER(I)]),
        "pqkv_pool_prefix_insert": (I, [P, P, I, P, I]),
        "pqkv_pool_cow": (I, [P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(I)]),
        "pqkv_copy_blocks": (I, [P, P, P, P, I, I, I, I, P, I, P, P]),
        "pqkv_block_record_bytes": (Z, [I, I, I]),
        "pqkv_swap_out": (I, [P, P, P, P, I, I, I, I, P, I, P, P, P]),
        "pqkv_swap_in": (I, [P, P, P, P, I, I, I, I, P, I, P, P, P]),
        "pqkv_paged_prefill_attention": (I, [P, I, I, I, I, P, P, P, P, P, I, I, I, I, P, I, P, ctypes.c_float,
                                             P, P, P]),
        "pqkv_paged_multi_query_decode_attention": (I, [P, I, I, I, I, P, P, P, P, I, I, I, I, P, I, P,
                                                        ctypes.c_float, I, P, P, Z, P, P]),
        "pqkv_read_probe": (I, [P, I, I, I, I, P, I, P, I, P, P, P]),
        "pqkv_set_decode_wait_limit_ns": (None, [ctypes.c_uint64]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib_handle: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libpqkv.so (loaded on first use; ImportError if not built)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


class _LazyLib:
    def __getattr__(self, name):
        return getattr(lib(), name)


_lib = _LazyLib()


def _check(func: str, status: int) -> None:
    if status != OK:
        raise PqkvError(func, status)


def _dev_ptr(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream_handle(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _dt_of(t: torch.Tensor, name: str) -> int:
    if t.dtype == torch.float16:
        return FP16
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError("%s must be float16 or bfloat16" % name)


def set_decode_wait_limit_ns(ns: int) -> None:
    """pqkv_set_decode_wait_limit_ns: limit of the decode and prefill kernels'
    waits for later launches (0 = the default 2 s); for tests of the timeout path."""
    _lib.pqkv_set_decode_wait_limit_ns(int(ns))


def version() -> int:
    return int(_lib.pqkv_version())


def cache_layout(kv_dtype: int, num_blocks: int, num_kv_heads: int, head_dim: int) -> Tuple[int, int, int, int]:
    """Byte sizes of (cache, scales, outliers_idx, outliers_val)."""
    out = (ctypes.c_size_t * 4)()
    _check("pqkv_cache_layout", _lib.pqkv_cache_layout(kv_dtype, num_blocks, num_kv_heads, head_dim, out))
    return tuple(int(x) for x in out)


@dataclasses.dataclass
class KVCache:
    """Device arrays of one layer's paged cache (uint8 views; None if unused)."""
    kv_dtype: int
    num_blocks: int
    num_kv_heads: int
    head_dim: int
    cache: torch.Tensor
    scales: Optional[torch.Tensor]
    outliers_idx: Optional[torch.Tensor]
    outliers_val: Optional[torch.Tensor]

    def arrays(self):
        return self.cache, self.scales, self.outliers_idx, self.outliers_val


def allocate_cache(kv_dtype: int, num_blocks: int, num_kv_heads: int, head_dim: int,
                   device="cuda", fill: Optional[int] = None) -> KVCache:
    """Allocate the cache arrays with torch (optionally filled with a byte)."""
    sizes = cache_layout(kv_dtype, num_blocks, num_kv_heads, head_dim)
    mk = (lambda n: torch.empty(n, dtype=torch.uint8, device=device)) if fill is None else \
        (lambda n: torch.full((n,), fill, dtype=torch.uint8, device=device))
    arrs = [mk(n) if n else None for n in sizes]
    return KVCache(kv_dtype, num_blocks, num_kv_heads, head_dim, *arrs)


def kv_cache_write(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, cache: KVCache,
                   err_flag: torch.Tensor, stream=None) -> None:
    """pqkv_kv_cache_write: k, v [T][Hkv][D] fp16/bf16, slot_mapping int32 [T]."""
    T = k.shape[0]
    if k.shape != (T, cache.num_kv_heads, cache.head_dim) or v.shape != k.shape:
        raise ValueError("k and v must be [T][num_kv_heads][head_dim]")
    if slot_mapping.dtype != torch.int32 or slot_mapping.numel() != T:
        raise ValueError("slot_mapping must be int32 [T]")
    if err_flag.dtype != torch.int32:
        raise ValueError("err_flag must be int32")
    st = _lib.pqkv_kv_cache_write(
        _dev_ptr(k, "k"), _dev_ptr(v, "v"), _dt_of(k, "k"), T, _dev_ptr(slot_mapping, "slot_mapping"),
        _dev_ptr(cache.cache, "cache"), _dev_ptr(cache.scales, "scales"),
        _dev_ptr(cache.outliers_idx, "outliers_idx"), _dev_ptr(cache.outliers_val, "outliers_val"),
        cache.kv_dtype, cache.num_blocks, cache.num_kv_heads, cache.head_dim,
        _dev_ptr(err_flag, "err_flag"), _stream_handle(stream, k.device))
    _check("pqkv_kv_cache_write", st)


def decode_workspace_bytes(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                           max_blocks_per_seq: int, split_blocks: int = 0) -> int:
    n = int(_lib.pqkv_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim,
                                              max_blocks_per_seq, split_blocks))
    if n == 0:
        raise PqkvError("pqkv_decode_workspace_bytes", ERR_ARG)
    return n


def decode_workspace(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                     max_blocks_per_seq: int, split_blocks: int = 0, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the required size (torch allocation)."""
    n = decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, split_blocks)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def multi_query_decode_workspace(batch: int, q_len: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                                 max_blocks_per_seq: int, split_blocks: int = 0, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for paged_multi_query_decode_attention (torch allocation)."""
    n = int(_lib.pqkv_multi_query_decode_workspace_bytes(batch, q_len, num_q_heads, num_kv_heads, head_dim,
                                                         max_blocks_per_seq, split_blocks))
    if n == 0:
        raise PqkvError("pqkv_multi_query_decode_workspace_bytes", ERR_ARG)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check("pqkv_decode_workspace_init", _lib.pqkv_decode_workspace_init(
        _dev_ptr(workspace, "workspace"), workspace.numel(), _stream_handle(stream, workspace.device)))


def paged_decode_attention(q: torch.Tensor, cache: KVCache, block_tables: torch.Tensor,
                           seq_lens: torch.Tensor, scale: float, out: torch.Tensor,
                           workspace: torch.Tensor, err_flag: torch.Tensor,
                           split_blocks: int = 0, stream=None) -> None:
    """pqkv_paged_decode_attention: q, out [B][Hq][D]; block_tables int32 [B][max_blocks];
    seq_lens int32 [B]."""
    B, Hq, D = q.shape
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B][max_blocks_per_seq]")
    if seq_lens.dtype != torch.int32 or seq_lens.numel() != B:
        raise ValueError("seq_lens must be int32 [B]")
    st = _lib.pqkv_paged_decode_attention(
        _dev_ptr(q, "q"), _dt_of(q, "q"), B, Hq, _dev_ptr(cache.cache, "cache"),
        _dev_ptr(cache.scales, "scales"), _dev_ptr(cache.outliers_idx, "outliers_idx"),
        _dev_ptr(cache.outliers_val, "outliers_val"), cache.kv_dtype, cache.num_blocks,
        cache.num_kv_heads, cache.head_dim, _dev_ptr(block_tables, "block_tables"),
        block_tables.shape[1], _dev_ptr(seq_lens, "seq_lens"), ctypes.c_float(scale), split_blocks,
        _dev_ptr(out, "out"), _dev_ptr(workspace, "workspace"), workspace.numel(),
        _dev_ptr(err_flag, "err_flag"), _stream_handle(stream, q.device))
    _check("pqkv_paged_decode_attention", st)


def paged_multi_query_decode_attention(q: torch.Tensor, cache: KVCache, block_tables: torch.Tensor,
                                      seq_lens: torch.Tensor, scale: float, out: torch.Tensor,
                                      workspace: torch.Tensor, err_flag: torch.Tensor, split_blocks: int = 0,
                                      stream=None) -> None:
    """pqkv_paged_multi_query_decode_attention: q, out [B][q_len][Hq][D] (each sequence's last q_len
    positions); workspace from multi_query_decode_workspace(B, q_len, Hq, ...)."""
    B, k, Hq, D = q.shape
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B][max_blocks_per_seq]")
    if seq_lens.dtype != torch.int32 or seq_lens.numel() != B:
        raise ValueError("seq_lens must be int32 [B]")
    st = _lib.pqkv_paged_multi_query_decode_attention(
        _dev_ptr(q, "q"), _dt_of(q, "q"), B, k, Hq, _dev_ptr(cache.cache, "cache"),
        _dev_ptr(cache.scales, "scales"), _dev_ptr(cache.outliers_idx, "outliers_idx"),
        _dev_ptr(cache.outliers_val, "outliers_val"), cache.kv_dtype, cache.num_blocks,
        cache.num_kv_heads, cache.head_dim, _dev_ptr(block_tables, "block_tables"),
        block_tables.shape[1], _dev_ptr(seq_lens, "seq_lens"), ctypes.c_float(scale), split_blocks,
        _dev_ptr(out, "out"), _dev_ptr(workspace, "workspace"), workspace.numel(),
        _dev_ptr(err_flag, "err_flag"), _stream_handle(stream, q.device))
    _check("pqkv_paged_multi_query_decode_attention", st)


def paged_prefill_attention(q: torch.Tensor, cu_q_lens: torch.Tensor, max_q_len: int, cache: KVCache,
                            block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, out: torch.Tensor,
                            err_flag: torch.Tensor, stream=None) -> None:
    """pqkv_paged_prefill_attention: q, out [T][Hq][D]; cu_q_lens int32 [B + 1]; block_tables int32
    [B][max_blocks]; seq_lens int32 [B] (each sequence's query tokens are its last positions)."""
    T, Hq, D = q.shape
    B = seq_lens.numel()
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if cu_q_lens.dtype != torch.int32 or cu_q_lens.numel() != B + 1:
        raise ValueError("cu_q_lens must be int32 [B + 1]")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B][max_blocks_per_seq]")
    if seq_lens.dtype != torch.int32:
        raise ValueError("seq_lens must be int32 [B]")
    st = _lib.pqkv_paged_prefill_attention(
        _dev_ptr(q, "q"), _dt_of(q, "q"), B, max_q_len, Hq, _dev_ptr(cu_q_lens, "cu_q_lens"),
        _dev_ptr(cache.cache, "cache"), _dev_ptr(cache.scales, "scales"),
        _dev_ptr(cache.outliers_idx, "outliers_idx"), _dev_ptr(cache.outliers_val, "outliers_val"),
        cache.kv_dtype, cache.num_blocks, cache.num_kv_heads, cache.head_dim,
        _dev_ptr(block_tables, "block_tables"), block_tables.shape[1], _dev_ptr(seq_lens, "seq_lens"),
        ctypes.c_float(scale), _dev_ptr(out, "out"), _dev_ptr(err_flag, "err_flag"),
        _stream_handle(stream, q.device))
    _check("pqkv_paged_prefill_attention", st)


def encode(x: torch.Tensor, code_dtype: int, out: torch.Tensor, stream=None) -> None:
    """pqkv_encode: float32 -> one code per byte (FP8 E4M3 / E5M2 / E2M1)."""
    if x.dtype != torch.float32 or out.dtype != torch.uint8 or out.numel() != x.numel():
        raise ValueError("x must be float32 and out uint8 of the same size")
    _check("pqkv_encode", _lib.pqkv_encode(_dev_ptr(x, "x"), x.numel(), code_dtype, _dev_ptr(out, "out"),
                                           _stream_handle(stream, x.device)))


def read_probe(cache: KVCache, block_tables: torch.Tensor, seq_lens: torch.Tensor, checksum: torch.Tensor,
               err_flag: torch.Tensor, stream=None) -> None:
    """pqkv_read_probe: the decode's paged gather of K|V tiles without its math
    (a bandwidth measurement); checksum: device int32 [1] that the caller zeroes."""
    B = seq_lens.numel()
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B][max_blocks_per_seq]")
    if seq_lens.dtype != torch.int32:
        raise ValueError("seq_lens must be int32 [B]")
    if checksum.dtype != torch.int32 or checksum.numel() < 1:
        raise ValueError("checksum must be int32 [1]")
    _check("pqkv_read_probe", _lib.pqkv_read_probe(
        _dev_ptr(cache.cache, "cache"), cache.kv_dtype, cache.num_blocks, cache.num_kv_heads, cache.head_dim,
        _dev_ptr(block_tables, "block_tables"), block_tables.shape[1], _dev_ptr(seq_lens, "seq_lens"), B,
        _dev_ptr(checksum, "checksum"), _dev_ptr(err_flag, "err_flag"),
        _stream_handle(stream, cache.cache.device)))


def copy_blocks(cache: KVCache, pairs: torch.Tensor, err_flag: torch.Tensor, stream=None) -> None:
    """pqkv_copy_blocks: pairs int32 [n][2] (src, dst) on the device."""
    if pairs.dtype != torch.int32 or pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be int32 [n][2]")
    _check("pqkv_copy_blocks", _lib.pqkv_copy_blocks(
        _dev_ptr(cache.cache, "cache"), _dev_ptr(cache.scales, "scales"),
        _dev_ptr(cache.outliers_idx, "outliers_idx"), _dev_ptr(cache.outliers_val, "outliers_val"),
        cache.kv_dtype, cache.num_blocks, cache.num_kv_heads, cache.head_dim,
        _dev_ptr(pairs, "pairs"), pairs.shape[0], _dev_ptr(err_flag, "err_flag"),
        _stream_handle(stream, cache.cache.device)))


def block_record_bytes(kv_dtype: int, num_kv_heads: int, head_dim: int) -> int:
    n = int(_lib.pqkv_block_record_bytes(kv_dtype, num_kv_heads, head_dim))
    if n == 0:
        raise PqkvError("pqkv_block_record_bytes", ERR_ARG)
    return n


def _host_records(records: torch.Tensor, n: int, rec: int) -> int:
    if not isinstance(records, torch.Tensor) or records.is_cuda or not records.is_pinned():
        raise ValueError("records must be a pinned host tensor")
    if not records.is_contiguous() or records.numel() * records.element_size() < n * rec:
        raise ValueError("records must be contiguous with room for %d records of %d bytes" % (n, rec))
    return records.data_ptr()


def swap_out(cache: KVCache, block_ids: torch.Tensor, records: torch.Tensor, err_flag: torch.Tensor,
             stream=None) -> None:
    """pqkv_swap_out: block_ids int32 [n] (device) -> records (pinned host, n records)."""
    if block_ids.dtype != torch.int32 or block_ids.dim() != 1:
        raise ValueError("block_ids must be int32 [n]")
    n = block_ids.numel()
    rec = block_record_bytes(cache.kv_dtype, cache.num_kv_heads, cache.head_dim)
    _check("pqkv_swap_out", _lib.pqkv_swap_out(
        _dev_ptr(cache.cache, "cache"), _dev_ptr(cache.scales, "scales"),
        _dev_ptr(cache.outliers_idx, "outliers_idx"), _dev_ptr(cache.outliers_val, "outliers_val"),
        cache.kv_dtype, cache.num_blocks, cache.num_kv_heads, cache.head_dim,
        _dev_ptr(block_ids, "block_ids"), n, _host_records(records, n, rec), _dev_ptr(err_flag, "err_flag"),
        _stream_handle(stream, cache.cache.device)))


def swap_in(cache: KVCache, block_ids: torch.Tensor, records: torch.Tensor, err_flag: torch.Tensor,
            stream=None) -> None:
    """pqkv_swap_in: records (pinned host, n records) -> blocks block_ids int32 [n] (device)."""
    if block_ids.dtype != torch.int32 or block_ids.dim() != 1:
        raise ValueError("block_ids must be int32 [n]")
    n = block_ids.numel()
    rec = block_record_bytes(cache.kv_dtype, cache.num_kv_heads, cache.head_dim)
    _check("pqkv_swap_in", _lib.pqkv_swap_in(
        _dev_ptr(cache.cache, "cache"), _dev_ptr(cache.scales, "scales"),
        _dev_ptr(cache.outliers_idx, "outliers_idx"), _dev_ptr(cache.outliers_val, "outliers_val"),
        cache.kv_dtype, cache.num_blocks, cache.num_kv_heads, cache.head_dim,
        _dev_ptr(block_ids, "block_ids"), n, _host_records(records, n, rec), _dev_ptr(err_flag, "err_flag"),
        _stream_handle(stream, cache.cache.device)))


class BlockPool:
    """Host block-pool allocator (pqkv_pool_*): physical ids with reference counts."""

    def __init__(self, num_blocks: int):
        h = ctypes.c_void_p()
        _check("pqkv_pool_create", _lib.pqkv_pool_create(num_blocks, ctypes.byref(h)))
        self._h = h
        self.num_blocks = num_blocks

    def close(self) -> None:
        if self._h:
            _lib.pqkv_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _ids(ids) -> np.ndarray:
        return np.ascontiguousarray(np.asarray(ids, dtype=np.int32).ravel())

    def alloc(self, n: int) -> np.ndarray:
        out = np.empty(n, dtype=np.int32)
        _check("pqkv_pool_alloc", _lib.pqkv_pool_alloc(self._h, n, out.ctypes.data))
        return out

    def share(self, ids) -> None:
        a = self._ids(ids)
        _check("pqkv_pool_share", _lib.pqkv_pool_share(self._h, a.ctypes.data, a.size))

    def free(self, ids) -> None:
        a = self._ids(ids)
        _check("pqkv_pool_free", _lib.pqkv_pool_free(self._h, a.ctypes.data, a.size))

    @property
    def num_free(self) -> int:
        return int(_lib.pqkv_pool_num_free(self._h))

    def refcount(self, block_id: int) -> int:
        return int(_lib.pqkv_pool_refcount(self._h, block_id))

    @property
    def num_evictable(self) -> int:
        return int(_lib.pqkv_pool_num_evictable(self._h))

    @property
    def num_cached(self) -> int:
        return int(_lib.pqkv_pool_num_cached(self._h))

    def prefix_lookup(self, token_ids) -> np.ndarray:
        """Ids of the longest cached prefix of token_ids (whole blocks); each gains a reference."""
        t = self._ids(token_ids)
        out = np.empty(max(1, t.size // 16), dtype=np.int32)
        hit = ctypes.c_int(0)
        _check("pqkv_pool_prefix_lookup", _lib.pqkv_pool_prefix_lookup(
            self._h, t.ctypes.data, t.size, out.ctypes.data, ctypes.byref(hit)))
        return out[:hit.value].copy()

    def prefix_insert(self, token_ids, ids) -> None:
        t = self._ids(token_ids)
        a = self._ids(ids)
        _check("pqkv_pool_prefix_insert", _lib.pqkv_pool_prefix_insert(
            self._h, t.ctypes.data, t.size, a.ctypes.data, a.size))

    def cow(self, block_id: int) -> Tuple[int, bool]:
        """(block to write into, whether block_id must be copied into it first)."""
        new = ctypes.c_int32(-1)
        need = ctypes.c_int(0)
        _check("pqkv_pool_cow", _lib.pqkv_pool_cow(self._h, block_id, ctypes.byref(new), ctypes.byref(need)))
        return int(new.value), bool(need.value)


def build_slot_mapping(block_tables: np.ndarray, start_pos: Sequence[int], num_new: Sequence[int]) -> np.ndarray:
    """pqkv_build_slot_mapping on host arrays; returns int32 slots."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sp = np.ascontiguousarray(start_pos, dtype=np.int32)
    nn = np.ascontiguousarray(num_new, dtype=np.int32)
    out = np.empty(int(nn.sum()), dtype=np.int32)
    _check("pqkv_build_slot_mapping", _lib.pqkv_build_slot_mapping(
        bt.ctypes.data, bt.shape[0], bt.shape[1], sp.ctypes.data, nn.ctypes.data, out.ctypes.data))
    return out
