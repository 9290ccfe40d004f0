"""CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It wraps ``dsa_oracle.c`` (plain C,
double accumulation, one pass per definition) through ctypes and takes numpy
arrays.  It shares no code with the CUDA library: no headers, helpers or
constants; the two meet only in the seeded input generator
(``long_context_sparse_fp8_b200.workloads``), which holds no DSA arithmetic.

Sources of each definition (page title and section):
  * indexer score / top-k / sparse attention: "SGLang Day-0 support for
    DeepSeek-V3.2" (winzheng.jp review), section "DeepSeek Sparse Attention";
    "DeepSeek-V3.2-Exp DSA deployment guide" (m.nxbn.cn) sections 1, 3.1, 5.1.
  * bf16 q with a bf16 or fp8 KV cache: "DeepSeek V3.2 usage guide" (SGLang
    docs), attention-kernel section.
  * cache writes (the page-64 key & key_scale cache, the token-level KV cache,
    FP8 storage): "SGLang Day-0 support for DeepSeek-V3.2", sections "DeepSeek
    Sparse Attention" and "Future work"; deployment guide section 3.1.

Dtype codes: 0 = fp32, 1 = bf16 (raw uint16 bits), 2 = fp8 e4m3 (raw bytes).
Parity pins for every function live in tests/test_oracle_pins.py; none of the
functions here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")

F32, BF16, E4M3 = 0, 1, 2
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into oracle/_build/liboracle.so (gcc, -O2, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared",
             "-fPIC", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_double.restype = dbl
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = dbl
            lib.oracle_indexer_logits.argtypes = [P, i32, P, P, i32, i32, P, i32, P, i32, P, i32,
                                                  i32, P, P, P, i64, P, i64]
            lib.oracle_indexer_logits.restype = i32
            lib.oracle_topk.argtypes = [P, i64, i32, P, P, P, i64, i32, P]
            lib.oracle_topk.restype = i32
            lib.oracle_sparse_mla.argtypes = [P, i32, i32, i32, i32, dbl, P, i32, P, i32, P, i32,
                                              i32, P, P, P, i32, P, i64, P, P]
            lib.oracle_sparse_mla.restype = i32
            lib.oracle_num_threads.restype = i32
            lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
            lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
            lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
            lib.oracle_cache_store.argtypes = [P, i32, i64, i32, P, P, i32, P, i64]
            lib.oracle_cache_store.restype = i32
            _lib = lib
    return _lib


def _c(a, dtype=None):
    """Contiguous numpy array (optionally cast) that stays alive with its pointer."""
    a = np.ascontiguousarray(a if dtype is None else np.asarray(a, dtype=dtype))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def e4m3_to_double(code: int) -> float:
    return float(_load().oracle_e4m3_to_double(code))


def bf16_to_double(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(bits))


def _rows(rows, total_q):
    if rows is None:
        rows = np.arange(total_q, dtype=np.int64)
    return _c(rows, np.int64)


def indexer_logits(q, q_dtype, q_scale, w, heads, dim, k_data, k_dtype, k_scale, page_size,
                   block_table, cu_q, seq_lens, ld, rows=None):
    """I[rows[r], s] for s <= pos, -inf beyond; returns float32 [len(rows), ld]."""
    lib = _load()
    cu_q = _c(cu_q, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    rows = _rows(rows, int(cu_q[-1]))
    q, w, k_data = _c(q), _c(w, np.float32), _c(k_data)
    q_scale = None if q_scale is None else _c(q_scale, np.float32)
    k_scale = None if k_scale is None else _c(k_scale, np.float32)
    bt = _c(block_table, np.int32)
    out = np.empty((len(rows), ld), dtype=np.float32)
    rc = lib.oracle_indexer_logits(_ptr(q), q_dtype, _ptr(q_scale), _ptr(w), heads, dim,
                                   _ptr(k_data), k_dtype, _ptr(k_scale), page_size, _ptr(bt),
                                   bt.shape[1], len(seq_lens), _ptr(cu_q), _ptr(seq_lens),
                                   _ptr(rows), len(rows), _ptr(out), ld)
    if rc != 0:
        raise ValueError("oracle_indexer_logits: malformed batch or table")
    return out


def topk(logits, cu_q, seq_lens, k, rows=None):
    """Selected positions per row, ascending, -1 padded; int32 [len(rows), k].

    ``logits[r]`` holds the scores of query row ``rows[r]``.
    """
    lib = _load()
    cu_q = _c(cu_q, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    rows = _rows(rows, int(cu_q[-1]))
    logits = _c(logits, np.float32)
    idx = np.empty((len(rows), k), dtype=np.int32)
    rc = lib.oracle_topk(_ptr(logits), logits.shape[1], len(seq_lens), _ptr(cu_q),
                         _ptr(seq_lens), _ptr(rows), len(rows), k, _ptr(idx))
    if rc != 0:
        raise ValueError("oracle_topk: malformed batch")
    return idx


def sparse_mla(q, q_dtype, heads, d_qk, d_v, softmax_scale, kv, kv_dtype, kv_scale, page_size,
               block_table, cu_q, seq_lens, idx, rows=None):
    """(out float32 [len(rows), heads, d_v], lse float32 [len(rows), heads]).

    ``idx[r]`` lists the selected positions of query row ``rows[r]``.
    """
    lib = _load()
    cu_q = _c(cu_q, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    rows = _rows(rows, int(cu_q[-1]))
    q, kv = _c(q), _c(kv)
    kv_scale = None if kv_scale is None else _c(kv_scale, np.float32)
    bt = _c(block_table, np.int32)
    idx = _c(idx, np.int32)
    out = np.empty((len(rows), heads, d_v), dtype=np.float32)
    lse = np.empty((len(rows), heads), dtype=np.float32)
    rc = lib.oracle_sparse_mla(_ptr(q), q_dtype, heads, d_qk, d_v, float(softmax_scale),
                               _ptr(kv), kv_dtype, _ptr(kv_scale), page_size, _ptr(bt),
                               bt.shape[1], len(seq_lens), _ptr(cu_q), _ptr(seq_lens),
                               _ptr(idx), idx.shape[1], _ptr(rows), len(rows), _ptr(out),
                               _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_sparse_mla: index outside [-1, pos] or malformed batch")
    return out, lse


def f32_to_e4m3(x: float) -> int:
    """One fp32 value to its e4m3 code (RNE, saturating at 448, sign kept)."""
    return int(_load().oracle_f32_to_e4m3(float(x)))


def f32_to_bf16(x: float) -> int:
    """One fp32 value to bf16 bits (RNE)."""
    return int(_load().oracle_f32_to_bf16(float(x)))


def cache_store(x, x_dtype, slot_mapping, cache_data, cache_dtype, cache_scale):
    """Writes the rows of ``x`` [n, dim] into copies of ``cache_data`` [num_rows, dim]
    (raw numpy of the cache dtype) and ``cache_scale`` [num_rows] (or None); returns
    (data, scale).  Row i goes to cache row ``slot_mapping[i]``; negative skips."""
    lib = _load()
    x = _c(x)
    n, dim = x.shape
    slots = _c(slot_mapping, np.int64)
    assert slots.shape == (n,)
    data = np.array(cache_data, copy=True, order="C")
    scale = None if cache_scale is None else np.array(cache_scale, dtype=np.float32, copy=True)
    if cache_dtype == E4M3 and scale is None:
        raise ValueError("an fp8 cache needs its scale array")
    rc = lib.oracle_cache_store(_ptr(x), x_dtype, n, dim, _ptr(slots), _ptr(data), cache_dtype,
                                _ptr(scale), data.shape[0])
    if rc != 0:
        raise ValueError("oracle_cache_store: slot outside [0, num_rows)")
    return data, scale
