"""Host-only checks of the C ABI: the library loads, exports every declared entry
point, and rejects bad arguments before touching the GPU (no device needed)."""
import ctypes
import os
import re

import pytest

import long_context_sparse_fp8_b200 as L
from long_context_sparse_fp8_b200 import dsa as D

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # an aligned non-NULL address; validation never dereferences it
FAKE2 = 0x20000


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = L.load_library()
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(D.EXPORTED)
    assert L.dsa_version() >= 100


def _batch(num_seqs=1, total_q=4, max_len=256):
    return D.DsaBatch(num_seqs, total_q, max_len, 0, FAKE, FAKE2)


def _cache(page_size=64, dim=128, dtype=D.DSA_FP8_E4M3, stride=4, pages=16, data=FAKE):
    return D.DsaPagedCache(data, None, FAKE2, pages, page_size, dim, stride, dtype)


def _status_msg():
    return L.load_library().dsa_last_error_message().decode()


def _indexer(batch, cache, q=FAKE, q_dtype=D.DSA_FP8_E4M3, heads=64, dim=128, ld=256, logits=FAKE,
             w=FAKE):
    lib = L.load_library()
    return lib.dsa_indexer_logits(q, q_dtype, None, w, heads, dim, ctypes.byref(cache),
                                  ctypes.byref(batch) if batch is not None else None, logits, ld,
                                  None)


@pytest.mark.parametrize("case,expect", [
    ("null_batch", D.DSA_ERR_INVALID_ARGUMENT),
    ("zero_seqs", D.DSA_ERR_INVALID_ARGUMENT),
    ("page_32", D.DSA_ERR_UNSUPPORTED),
    ("misaligned_q", D.DSA_ERR_INVALID_ARGUMENT),
    ("null_w", D.DSA_ERR_INVALID_ARGUMENT),
    ("short_ld", D.DSA_ERR_INVALID_ARGUMENT),
    ("fp8_heads_32", D.DSA_ERR_UNSUPPORTED),
    ("dtype_mismatch", D.DSA_ERR_UNSUPPORTED),
    ("short_block_table", D.DSA_ERR_INVALID_ARGUMENT),
    ("bf16_indexer", D.DSA_ERR_UNSUPPORTED),
])
def test_indexer_rejects_bad_arguments(case, expect):
    b, c = _batch(), _cache()
    kw = {}
    if case == "null_batch":
        b = None
    elif case == "zero_seqs":
        b = _batch(num_seqs=0)
    elif case == "page_32":
        c = _cache(page_size=32, stride=8)
    elif case == "misaligned_q":
        kw["q"] = FAKE + 4
    elif case == "null_w":
        kw["w"] = None
    elif case == "short_ld":
        kw["ld"] = 128
    elif case == "fp8_heads_32":
        kw["heads"] = 32
    elif case == "dtype_mismatch":
        kw["q_dtype"] = D.DSA_F32
    elif case == "short_block_table":
        c = _cache(stride=3)
    elif case == "bf16_indexer":
        c = _cache(dtype=D.DSA_BF16)
        kw["q_dtype"] = D.DSA_BF16
    st = _indexer(b, c, **kw)
    assert st == expect, (case, st, _status_msg())
    assert _status_msg()


def test_topk_rejects_bad_arguments():
    lib = L.load_library()
    b = _batch()
    assert lib.dsa_topk(FAKE, 256, ctypes.byref(b), 0, FAKE2, None) == D.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(FAKE, 255, ctypes.byref(b), 8, FAKE2, None) == D.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(None, 256, ctypes.byref(b), 8, FAKE2, None) == D.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(FAKE, 256, ctypes.byref(b), 70000, FAKE2, None) == \
        D.DSA_ERR_INVALID_ARGUMENT


def _mla(fn="dsa_sparse_mla_prefill", q_dtype=D.DSA_BF16, heads=128, d_qk=576, d_v=512,
         kv=None, out_dtype=D.DSA_BF16, k=2048, scale=0.07, ws=None, ws_bytes=0, total_q=4):
    lib = L.load_library()
    b = _batch(total_q=total_q)
    kv = kv or _cache(page_size=1, dim=576, dtype=D.DSA_BF16, stride=256, pages=1024)
    args = [FAKE, q_dtype, heads, d_qk, d_v, scale, ctypes.byref(kv), ctypes.byref(b), FAKE2, k,
            FAKE, out_dtype, None]
    if fn == "dsa_sparse_mla_decode":
        args += [ws, ws_bytes]
    return getattr(lib, fn)(*args, None)


def test_mla_rejects_bad_arguments():
    assert _mla(heads=64) == D.DSA_ERR_UNSUPPORTED
    assert _mla(out_dtype=D.DSA_F32) == D.DSA_ERR_UNSUPPORTED
    assert _mla(d_v=600) == D.DSA_ERR_INVALID_ARGUMENT
    assert _mla(k=0) == D.DSA_ERR_INVALID_ARGUMENT
    assert _mla(scale=0.0) == D.DSA_ERR_INVALID_ARGUMENT
    assert _mla(kv=_cache(page_size=64, dim=576, dtype=D.DSA_BF16, stride=4)) == \
        D.DSA_ERR_UNSUPPORTED
    assert _mla(kv=_cache(page_size=1, dim=576, dtype=D.DSA_BF16, stride=256, data=FAKE + 8)) == \
        D.DSA_ERR_INVALID_ARGUMENT
    assert _mla(q_dtype=D.DSA_FP8_E4M3) == D.DSA_ERR_UNSUPPORTED


def test_mla_decode_needs_its_workspace():
    lib = L.load_library()
    need = lib.dsa_sparse_mla_decode_workspace_size(32, 128, 512, 2048)
    assert need > 0
    st = _mla("dsa_sparse_mla_decode", ws=FAKE, ws_bytes=need - 1, total_q=32)
    assert st == D.DSA_ERR_WORKSPACE_TOO_SMALL, _status_msg()
    st = _mla("dsa_sparse_mla_decode", ws=None, ws_bytes=need, total_q=32)
    assert st == D.DSA_ERR_INVALID_ARGUMENT


def test_decode_workspace_is_checked_before_launch():
    lib = L.load_library()
    b = _batch(num_seqs=32, total_q=32, max_len=8192)
    need = lib.dsa_decode_workspace_size(ctypes.byref(b), 2048, 128, 512)
    assert need >= 32 * 8192 * 4 + 32 * 2048 * 4
    kc = _cache(stride=128)
    kv = _cache(page_size=1, dim=576, dtype=D.DSA_BF16, stride=8192, pages=32 * 8192)
    st = lib.dsa_decode(FAKE, D.DSA_FP8_E4M3, None, FAKE, 64, 128, ctypes.byref(kc), 2048, FAKE,
                        D.DSA_BF16, 128, 576, 512, 0.07, ctypes.byref(kv), ctypes.byref(b), None,
                        FAKE2, D.DSA_BF16, None, FAKE, need - 16, None)
    assert st == D.DSA_ERR_WORKSPACE_TOO_SMALL


def test_status_strings():
    lib = L.load_library()
    for st in range(6):
        assert lib.dsa_status_string(st).decode().startswith("DSA_")


@pytest.mark.parametrize("case,expect", [
    ("neg_n", D.DSA_ERR_INVALID_ARGUMENT),
    ("x_fp8", D.DSA_ERR_UNSUPPORTED),
    ("dim_100", D.DSA_ERR_UNSUPPORTED),
    ("dim_2048", D.DSA_ERR_UNSUPPORTED),
    ("misaligned_x", D.DSA_ERR_INVALID_ARGUMENT),
    ("null_slots", D.DSA_ERR_INVALID_ARGUMENT),
    ("fp8_no_scale", D.DSA_ERR_INVALID_ARGUMENT),
    ("zero_rows", D.DSA_ERR_INVALID_ARGUMENT),
    ("bad_cache_dtype", D.DSA_ERR_INVALID_ARGUMENT),
])
def test_cache_store_rejects_bad_arguments(case, expect):
    a = dict(x=FAKE, xt=D.DSA_BF16, n=4, dim=128, slots=FAKE2, data=FAKE, ct=D.DSA_FP8_E4M3,
             scale=FAKE2, rows=256)
    a.update({"neg_n": dict(n=-1), "x_fp8": dict(xt=D.DSA_FP8_E4M3), "dim_100": dict(dim=100),
              "dim_2048": dict(dim=2048), "misaligned_x": dict(x=FAKE + 4),
              "null_slots": dict(slots=None), "fp8_no_scale": dict(scale=None),
              "zero_rows": dict(rows=0), "bad_cache_dtype": dict(ct=9)}[case])
    st = L.load_library().dsa_cache_store(a["x"], a["xt"], a["n"], a["dim"], a["slots"], a["data"],
                                          a["ct"], a["scale"], a["rows"], None)
    assert st == expect, _status_msg()
    assert _status_msg()


def test_cache_store_empty_is_a_no_op():
    assert L.load_library().dsa_cache_store(None, D.DSA_BF16, 0, 128, None, None,
                                            D.DSA_FP8_E4M3, None, 1, None) == D.DSA_OK


def test_indexer_topk_checks_its_workspace():
    lib = L.load_library()
    b = _batch(1, 8192, 32768)
    need = lib.dsa_indexer_topk_workspace_size(ctypes.byref(b))
    assert need == 592 * 32768 * 4                 # a 74 MB block: 4 rows x 148 SMs
    c = _cache()
    st = lib.dsa_indexer_topk(FAKE, D.DSA_FP8_E4M3, None, FAKE, 64, 128, ctypes.byref(c),
                              ctypes.byref(b), 2048, FAKE, FAKE2, need - 1, None)
    assert st == D.DSA_ERR_WORKSPACE_TOO_SMALL, _status_msg()
    st = lib.dsa_indexer_topk(FAKE, D.DSA_FP8_E4M3, None, FAKE, 64, 128, ctypes.byref(c),
                              ctypes.byref(b), 2048, FAKE, None, need, None)
    assert st == D.DSA_ERR_INVALID_ARGUMENT, _status_msg()
    small = _batch(1, 8, 300)
    assert lib.dsa_indexer_topk_workspace_size(ctypes.byref(small)) == 8 * 320 * 4
