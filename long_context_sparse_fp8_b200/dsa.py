"""Thin ctypes binding of libdsa (include/dsa.h).

Argument marshalling only: every function takes torch tensors (device memory owned
by the caller), turns them into pointers and sizes, and calls the C function of the
same name on the current CUDA stream.  A non-OK status raises :class:`DsaError`.
The binding fails loudly when libdsa.so is missing; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARGUMENT = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_WORKSPACE_TOO_SMALL = 3
DSA_ERR_CUDA = 4
DSA_ERR_DEVICE_CHECK = 5

DSA_F32 = 0
DSA_BF16 = 1
DSA_FP8_E4M3 = 2

EXPORTED = (
    "dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla_prefill",
    "dsa_sparse_mla_decode_workspace_size", "dsa_sparse_mla_decode",
    "dsa_sparse_mla_decode_noalloc",
    "dsa_cache_store",
    "dsa_indexer_topk_workspace_size", "dsa_indexer_topk",
    "dsa_decode_workspace_size", "dsa_decode", "dsa_device_check", "dsa_last_error_message",
    "dsa_status_string", "dsa_version",
)

_TORCH_TO_DSA = {torch.float32: DSA_F32, torch.bfloat16: DSA_BF16,
                 torch.float8_e4m3fn: DSA_FP8_E4M3}


class DsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


class DsaBatch(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_q", ctypes.c_int32),
                ("max_seq_len", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("cu_q", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p)]


class DsaPagedCache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("num_pages", ctypes.c_int64),
                ("page_size", ctypes.c_int32), ("dim", ctypes.c_int32),
                ("bt_stride", ctypes.c_int32), ("dtype", ctypes.c_int)]


_lib = None


def load_library(path: str = _LIB_PATH) -> ctypes.CDLL:
    """Loads libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libdsa.so not found at {path}; run long_context_sparse_fp8_b200/_build.py")
    lib = ctypes.CDLL(path)
    P, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                            ctypes.c_float)
    BP, CP = ctypes.POINTER(DsaBatch), ctypes.POINTER(DsaPagedCache)
    sig = {
        "dsa_indexer_logits": ([P, ctypes.c_int, P, P, i32, i32, CP, BP, P, i64, P], ctypes.c_int),
        "dsa_topk": ([P, i64, BP, i32, P, P], ctypes.c_int),
        "dsa_sparse_mla_prefill": ([P, ctypes.c_int, i32, i32, i32, f32, CP, BP, P, i32, P,
                                    ctypes.c_int, P, P], ctypes.c_int),
        "dsa_sparse_mla_decode_workspace_size": ([i32, i32, i32, i32], sz),
        "dsa_sparse_mla_decode": ([P, ctypes.c_int, i32, i32, i32, f32, CP, BP, P, i32, P,
                                   ctypes.c_int, P, P, sz, P], ctypes.c_int),
        "dsa_sparse_mla_decode_noalloc": ([P, ctypes.c_int, i32, i32, i32, f32, CP, BP, P, i32,
                                           P, ctypes.c_int, P, P], ctypes.c_int),
        "dsa_decode_workspace_size": ([BP, i32, i32, i32], sz),
        "dsa_decode": ([P, ctypes.c_int, P, P, i32, i32, CP, i32, P, ctypes.c_int, i32, i32, i32,
                        f32, CP, BP, P, P, ctypes.c_int, P, P, sz, P], ctypes.c_int),
        "dsa_cache_store": ([P, ctypes.c_int, i32, i32, P, P, ctypes.c_int, P, i64, P],
                            ctypes.c_int),
        "dsa_indexer_topk_workspace_size": ([BP], sz),
        "dsa_indexer_topk": ([P, ctypes.c_int, P, P, i32, i32, CP, BP, i32, P, P, sz, P],
                             ctypes.c_int),
        "dsa_device_check": ([P, ctypes.POINTER(i32), i32], ctypes.c_int),
        "dsa_last_error_message": ([], ctypes.c_char_p),
        "dsa_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "dsa_version": ([], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _status_name(st: int) -> str:
    try:
        return load_library().dsa_status_string(st).decode()
    except Exception:  # pragma: no cover
        return f"status {st}"


def _check(st: int):
    if st != DSA_OK:
        raise DsaError(st, load_library().dsa_last_error_message().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def dtype_code(t: torch.Tensor) -> int:
    return _TORCH_TO_DSA[t.dtype]


@dataclass
class Batch:
    """A ragged batch: device ``cu_q [B+1]`` and ``seq_lens [B]`` plus host bounds."""
    cu_q: torch.Tensor
    seq_lens: torch.Tensor
    total_q: int
    max_seq_len: int

    def c(self) -> DsaBatch:
        return DsaBatch(int(self.seq_lens.numel()), int(self.total_q), int(self.max_seq_len), 0,
                        _ptr(self.cu_q), _ptr(self.seq_lens))


@dataclass
class PagedCache:
    """``data [num_pages, page_size, dim]`` (or ``[num_slots, dim]`` for page size 1),
    optional per-token ``scale``, and ``block_table [B, bt_stride]``."""
    data: torch.Tensor
    block_table: torch.Tensor
    page_size: int
    scale: Optional[torch.Tensor] = None

    def c(self) -> DsaPagedCache:
        dim = int(self.data.shape[-1])
        num_pages = int(self.data.numel() // (dim * self.page_size))
        return DsaPagedCache(_ptr(self.data), _ptr(self.scale), _ptr(self.block_table), num_pages,
                             self.page_size, dim, int(self.block_table.shape[1]),
                             dtype_code(self.data))


def dsa_indexer_logits(q, q_scale, w, k_cache: PagedCache, batch: Batch, logits, stream=None):
    heads, dim = int(q.shape[-2]), int(q.shape[-1])
    kc, bc = k_cache.c(), batch.c()
    _check(load_library().dsa_indexer_logits(
        _ptr(q), dtype_code(q), _ptr(q_scale), _ptr(w), heads, dim, ctypes.byref(kc),
        ctypes.byref(bc), _ptr(logits), int(logits.stride(0)), _stream(stream)))
    return logits


def dsa_topk(logits, batch: Batch, k: int, idx, stream=None):
    bc = batch.c()
    _check(load_library().dsa_topk(_ptr(logits), int(logits.stride(0)), ctypes.byref(bc), int(k),
                                   _ptr(idx), _stream(stream)))
    return idx


def dsa_sparse_mla_prefill(q, kv: PagedCache, batch: Batch, idx, d_v: int, softmax_scale: float,
                           out, lse=None, stream=None):
    heads, d_qk = int(q.shape[-2]), int(q.shape[-1])
    kc, bc = kv.c(), batch.c()
    _check(load_library().dsa_sparse_mla_prefill(
        _ptr(q), dtype_code(q), heads, d_qk, int(d_v), float(softmax_scale), ctypes.byref(kc),
        ctypes.byref(bc), _ptr(idx), int(idx.shape[-1]), _ptr(out), dtype_code(out), _ptr(lse),
        _stream(stream)))
    return out


def dsa_sparse_mla_decode_workspace_size(total_q: int, heads: int, d_v: int, k: int) -> int:
    return int(load_library().dsa_sparse_mla_decode_workspace_size(total_q, heads, d_v, k))


def dsa_sparse_mla_decode(q, kv: PagedCache, batch: Batch, idx, d_v: int, softmax_scale: float,
                          out, lse=None, workspace=None, stream=None):
    heads, d_qk = int(q.shape[-2]), int(q.shape[-1])
    kc, bc = kv.c(), batch.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().dsa_sparse_mla_decode(
        _ptr(q), dtype_code(q), heads, d_qk, int(d_v), float(softmax_scale), ctypes.byref(kc),
        ctypes.byref(bc), _ptr(idx), int(idx.shape[-1]), _ptr(out), dtype_code(out), _ptr(lse),
        _ptr(workspace), ws_bytes, _stream(stream)))
    return out


DSA_NOALLOC_SCRATCH_BYTES = 20 << 20


def dsa_sparse_mla_decode_noalloc(q, kv: PagedCache, batch: Batch, idx, d_v: int,
                                  softmax_scale: float, out, lse=None, stream=None):
    """dsa_sparse_mla_decode with the split partials in the library's fixed device
    array (no workspace argument; calls whose executions overlap on one device race)."""
    heads, d_qk = int(q.shape[-2]), int(q.shape[-1])
    kc, bc = kv.c(), batch.c()
    _check(load_library().dsa_sparse_mla_decode_noalloc(
        _ptr(q), dtype_code(q), heads, d_qk, int(d_v), float(softmax_scale), ctypes.byref(kc),
        ctypes.byref(bc), _ptr(idx), int(idx.shape[-1]), _ptr(out), dtype_code(out), _ptr(lse),
        _stream(stream)))
    return out


def dsa_decode_workspace_size(batch: Batch, k: int, heads: int, d_v: int) -> int:
    bc = batch.c()
    return int(load_library().dsa_decode_workspace_size(ctypes.byref(bc), k, heads, d_v))


def dsa_decode(q_idx, q_idx_scale, w, k_cache: PagedCache, k: int, q, kv: PagedCache,
               batch: Batch, d_v: int, softmax_scale: float, out, lse=None, idx_out=None,
               workspace=None, stream=None):
    idx_heads, idx_dim = int(q_idx.shape[-2]), int(q_idx.shape[-1])
    heads, d_qk = int(q.shape[-2]), int(q.shape[-1])
    kc, vc, bc = k_cache.c(), kv.c(), batch.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().dsa_decode(
        _ptr(q_idx), dtype_code(q_idx), _ptr(q_idx_scale), _ptr(w), idx_heads, idx_dim,
        ctypes.byref(kc), int(k), _ptr(q), dtype_code(q), heads, d_qk, int(d_v),
        float(softmax_scale), ctypes.byref(vc), ctypes.byref(bc), _ptr(idx_out), _ptr(out),
        dtype_code(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def dsa_indexer_topk_workspace_size(batch: Batch) -> int:
    bc = batch.c()
    return int(load_library().dsa_indexer_topk_workspace_size(ctypes.byref(bc)))


def dsa_indexer_topk(q, q_scale, w, k_cache: PagedCache, batch: Batch, k: int, idx,
                     workspace=None, stream=None):
    """Indexer + top-k over L2-sized blocks of query rows (no [T][L] logits); ``idx``
    [T, k] int32 receives the same lists as dsa_indexer_logits + dsa_topk.  Without a
    ``workspace`` (uint8, dsa_indexer_topk_workspace_size bytes) one is allocated."""
    heads, dim = int(q.shape[-2]), int(q.shape[-1])
    if workspace is None:
        n = dsa_indexer_topk_workspace_size(batch)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    kc, bc = k_cache.c(), batch.c()
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().dsa_indexer_topk(
        _ptr(q), dtype_code(q), _ptr(q_scale), _ptr(w), heads, dim, ctypes.byref(kc),
        ctypes.byref(bc), int(k), _ptr(idx), _ptr(workspace), ws_bytes, _stream(stream)))
    return idx


def dsa_cache_store(x, slot_mapping, cache_data, cache_scale=None, stream=None):
    """Writes the rows of ``x`` [n, dim] (fp32 / bf16) into ``cache_data`` (any shape
    whose last dim is ``dim``: [pages, page_size, dim] or [rows, dim]; fp8 e4m3, bf16
    or fp32) at flat rows ``slot_mapping`` [n] int64 (negative: skipped); an fp8 cache
    also gets its per-token ``cache_scale`` (amax / 448)."""
    n, dim = int(x.shape[0]), int(x.shape[-1])
    num_rows = cache_data.numel() // dim
    _check(load_library().dsa_cache_store(
        _ptr(x), dtype_code(x), n, dim, _ptr(slot_mapping), _ptr(cache_data),
        dtype_code(cache_data), _ptr(cache_scale), int(num_rows), _stream(stream)))
    return cache_data


def dsa_device_check(reset: bool = True, stream=None) -> int:
    """Synchronises the stream and returns the device check code (0 = clean)."""
    code = ctypes.c_int32(0)
    st = load_library().dsa_device_check(_stream(stream), ctypes.byref(code), int(reset))
    if st not in (DSA_OK, DSA_ERR_DEVICE_CHECK):
        _check(st)
    return int(code.value)


def dsa_version() -> int:
    return int(load_library().dsa_version())
