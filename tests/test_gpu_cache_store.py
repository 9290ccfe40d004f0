"""GPU parity of dsa_cache_store against the CPU oracle: every byte of every cache
row (codes and scales) must be identical -- the FP8 codes are integer decisions
both sides take from the same fp32 quotient."""
import numpy as np
import pytest
import torch

import long_context_sparse_fp8_b200 as L
from long_context_sparse_fp8_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu

_CODE = {torch.float32: O.F32, torch.bfloat16: O.BF16, torch.float8_e4m3fn: O.E4M3}


def _raw(t):
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def _store_and_compare(x, slots, data, scale):
    """Runs the GPU store and the oracle on copies of the same cache; compares all bytes."""
    dim = x.shape[-1]
    before_d = _raw(data).reshape(-1, dim).copy()
    before_s = None if scale is None else _raw(scale).reshape(-1).copy()
    L.dsa_cache_store(x, slots, data, scale)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    want_d, want_s = O.cache_store(_raw(x), _CODE[x.dtype], slots.cpu().numpy(), before_d,
                                   _CODE[data.dtype], before_s)
    got_d = _raw(data).reshape(-1, dim)
    bad = np.nonzero(np.any(got_d != want_d, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:5]}"
    if scale is not None:
        assert np.array_equal(_raw(scale).reshape(-1).view(np.uint32), want_s.view(np.uint32))


@pytest.mark.parametrize("n,skip", [(1, 0), (37, 5), (20000, 0), (4097, 3)])
def test_fp8_caches_match_oracle(n, skip):
    wl = W.make_store(W.StoreSpec(name="t", n_tokens=n, skip_every=skip, seed=50 + n), "cuda")
    _store_and_compare(wl.k_new, wl.k_slots, wl.k_pages, wl.k_scale)
    _store_and_compare(wl.kv_new, wl.kv_slots, wl.kv, wl.kv_scale)


def test_full_prompt_128k_matches_oracle():
    wl = W.make_store(W.store_prompt_128k(), "cuda")
    _store_and_compare(wl.k_new, wl.k_slots, wl.k_pages, wl.k_scale)
    _store_and_compare(wl.kv_new, wl.kv_slots, wl.kv, wl.kv_scale)


@pytest.mark.parametrize("x_dtype,kv_fp8", [("f32", True), ("f32", False), ("bf16", False)])
def test_other_dtypes_match_oracle(x_dtype, kv_fp8):
    wl = W.make_store(W.StoreSpec(name="t", n_tokens=3000, x_dtype=x_dtype, kv_fp8=kv_fp8,
                                  skip_every=7, seed=61), "cuda")
    _store_and_compare(wl.kv_new, wl.kv_slots, wl.kv, wl.kv_scale)
    f32 = torch.full((wl.kv.shape[0], wl.kv.shape[1]), 7.0, device="cuda")
    _store_and_compare(wl.kv_new, wl.kv_slots, f32, None)


def test_rounding_ties_subnormals_and_zero_rows():
    """Rows whose amax is 448 (scale exactly 1), so every element is its own
    quotient: all e4m3 midpoints (ties to even), one ulp either side, subnormal-range
    values, signed zeros; plus all-zero rows and rows of tiny values."""
    vals = np.array([O.e4m3_to_double(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    pool = np.concatenate([mids, np.nextafter(mids, np.float32(1e9)),
                           np.nextafter(mids, np.float32(0)), vals.astype(np.float32),
                           np.float32([2.0 ** -10, 3 * 2.0 ** -11, 1e-7, 0.0])])
    pool = np.concatenate([pool, -pool, np.float32([-0.0])])
    g = np.random.default_rng(3)
    dim, n = 576, 64
    x = g.choice(pool, (n, dim)).astype(np.float32)
    x[:, 0] = 448.0
    x[5] = 0.0
    x[6] = -0.0
    x[7] = g.standard_normal(dim).astype(np.float32) * np.float32(1e-30)
    xs = torch.from_numpy(x).cuda()
    slots = torch.arange(n, dtype=torch.int64, device="cuda")
    data = torch.zeros(n, dim, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
    scale = torch.zeros(n, device="cuda")
    _store_and_compare(xs, slots, data, scale)
    xb = xs.to(torch.bfloat16)
    _store_and_compare(xb, slots, data, scale)


def test_slot_past_the_end_is_recorded_and_skipped():
    wl = W.make_store(W.StoreSpec(name="t", n_tokens=300, seed=71), "cuda")
    slots = wl.kv_slots.clone()
    slots[10] = wl.kv.shape[0]              # one past the last row
    before = _raw(wl.kv).copy()
    L.dsa_cache_store(wl.kv_new, slots, wl.kv, wl.kv_scale)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 1        # DSA_CHECK_BAD_PAGE, then cleared
    assert L.dsa_device_check() == 0
    s = slots.cpu().numpy()
    good = np.delete(np.arange(300), 10)
    want, _ = O.cache_store(_raw(wl.kv_new)[good], O.BF16, s[good], before, O.E4M3,
                            np.full(wl.kv.shape[0], -1.0, np.float32))
    assert np.array_equal(_raw(wl.kv), want)


def test_stored_kv_feeds_decode_attention():
    """Keys and latent KV written by dsa_cache_store, then read by dsa_decode: the
    attention equals the oracle's on the stored caches."""
    import _helpers as H
    spec = W.Spec(name="st", seq_lens=[3000, 2100], nq=[1, 1], topk=2048, kv_fp8=True,
                  permute_tables=True, seed=81)
    wl = W.make(spec, device="cuda")
    # overwrite both caches with freshly stored rows for every position
    for b, Lb in enumerate(spec.seq_lens):
        pos = torch.arange(Lb, device="cuda")
        k_rows = torch.randn(Lb, spec.idx_dim, device="cuda").to(torch.bfloat16)
        kv_rows = torch.randn(Lb, spec.d_qk, device="cuda").to(torch.bfloat16)
        k_slot = (wl.k_block_table[b, pos // 64].long() * 64 + pos % 64)
        kv_slot = wl.kv_slot_table[b, pos].long()
        L.dsa_cache_store(k_rows, k_slot, wl.k_pages, wl.k_scale)
        L.dsa_cache_store(kv_rows, kv_slot, wl.kv, wl.kv_scale)
    torch.cuda.synchronize()
    rows = np.arange(spec.total_q)
    logits = H.run_indexer(wl)
    idx = H.run_topk(wl, logits)
    out, lse = H.run_mla(wl, idx, decode=True)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    pos = H.positions(wl)[rows]
    g_logits = logits.cpu().numpy()
    o_logits = H.oracle_logits(wl, rows)
    H.check_logits(g_logits, o_logits, pos)
    g_idx = idx.cpu().numpy()
    H.check_topk(g_idx, g_logits, o_logits, pos, spec.topk)
    o_ref, l_ref = H.oracle_mla(wl, g_idx, rows)
    H.check_mla(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, H.MLA_ATOL_BF16)


@pytest.mark.parametrize("dim", [128, 576])
def test_fp8_codes_on_rounding_boundaries(dim):
    """Rows whose elements sit next to e4m3 rounding boundaries (see _quant_cases):
    the last bit of each fp32 quotient x / scale decides the code, so any other way
    of forming the quotient shows up here as differing bytes."""
    import _quant_cases as QC
    x = torch.from_numpy(QC.boundary_rows(300, dim, seed=dim)).cuda()
    n = x.shape[0]
    slots = torch.randperm(n + 17, generator=torch.Generator().manual_seed(dim))[:n].cuda()
    data = torch.zeros(n + 17, dim, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
    scale = torch.full((n + 17,), -1.0, device="cuda")
    _store_and_compare(x, slots.to(torch.int64), data, scale)
