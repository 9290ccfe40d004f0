"""Shared plumbing of the parity tests: run the library on a workload, run the oracle
on chosen rows, and compare with the stated tolerances.

Tolerances (the problem statement's bars):
  * indexer logits: |gpu - oracle| <= 1e-3 * max(|oracle|, 1e-2 * max_row |oracle|);
  * top-k: the GPU set equals the oracle's top-k of the GPU's own logits exactly
    (integer work on identical inputs), and equals the oracle's top-k of the
    oracle's logits except for positions whose oracle score lies within 1e-3
    relative of the k-th score;
  * sparse MLA given the same index set: |gpu - oracle| <= 2e-2 for bf16 outputs,
    plus the half-ulp that rounding the output to bf16 costs by itself
    (|oracle| * 2^-8; it exceeds 2e-2 once |o| >= 8, which the x4 heavy-hitter
    rows produce); fp32 outputs (CUDA-core path) within 1e-4; lse within 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import long_context_sparse_fp8_b200 as L
from long_context_sparse_fp8_b200 import workloads as W
from oracle import oracle as O

LOGIT_RTOL = 1e-3
TIE_RTOL = 1e-3
MLA_ATOL_BF16 = 2e-2
MLA_ATOL_F32 = 1e-4
LSE_ATOL = 1e-2


def np_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def odt(t: torch.Tensor) -> int:
    return {torch.float32: O.F32, torch.bfloat16: O.BF16, torch.float8_e4m3fn: O.E4M3}[t.dtype]


def lib_args(wl: W.Workload):
    s = wl.spec
    batch = L.Batch(wl.cu_q, wl.seq_lens, s.total_q, s.max_seq_len)
    kc = L.PagedCache(wl.k_pages, wl.k_block_table, W.INDEXER_PAGE, wl.k_scale)
    kv = L.PagedCache(wl.kv, wl.kv_slot_table, 1, wl.kv_scale)
    return batch, kc, kv


def ld_for(wl: W.Workload) -> int:
    return (wl.spec.max_seq_len + 63) // 64 * 64


def positions(wl: W.Workload) -> np.ndarray:
    s = wl.spec
    pos = []
    for b in range(s.num_seqs):
        for i in range(s.nq[b]):
            pos.append(s.seq_lens[b] - s.nq[b] + i)
    return np.array(pos, dtype=np.int64)


def run_indexer(wl: W.Workload) -> torch.Tensor:
    batch, kc, _ = lib_args(wl)
    logits = torch.full((wl.spec.total_q, ld_for(wl)), float("nan"), device=wl.device)
    L.dsa_indexer_logits(wl.q_idx, None, wl.w, kc, batch, logits)
    return logits


def run_topk(wl: W.Workload, logits: torch.Tensor) -> torch.Tensor:
    batch, _, _ = lib_args(wl)
    idx = torch.full((wl.spec.total_q, wl.spec.topk), -7, dtype=torch.int32, device=wl.device)
    L.dsa_topk(logits, batch, wl.spec.topk, idx)
    return idx


def run_mla(wl: W.Workload, idx: torch.Tensor, decode: bool = False):
    s = wl.spec
    batch, _, kv = lib_args(wl)
    out_dt = torch.bfloat16 if s.mla_dtype == "bf16" else torch.float32
    out = torch.full((s.total_q, s.heads, s.d_v), float("nan"), dtype=out_dt, device=wl.device)
    lse = torch.full((s.total_q, s.heads), float("nan"), device=wl.device)
    if decode:
        n = L.dsa_sparse_mla_decode_workspace_size(s.total_q, s.heads, s.d_v, idx.shape[1])
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=wl.device)
        L.dsa_sparse_mla_decode(wl.q, kv, batch, idx, s.d_v, s.softmax_scale, out, lse, ws)
    else:
        L.dsa_sparse_mla_prefill(wl.q, kv, batch, idx, s.d_v, s.softmax_scale, out, lse)
    return out, lse


def oracle_logits(wl: W.Workload, rows: np.ndarray) -> np.ndarray:
    s = wl.spec
    return O.indexer_logits(np_bits(wl.q_idx), odt(wl.q_idx), None, np_bits(wl.w), s.idx_heads,
                            s.idx_dim, np_bits(wl.k_pages), odt(wl.k_pages),
                            None if wl.k_scale is None else np_bits(wl.k_scale), W.INDEXER_PAGE,
                            np_bits(wl.k_block_table), np_bits(wl.cu_q), np_bits(wl.seq_lens),
                            ld_for(wl), rows=rows)


def oracle_mla(wl: W.Workload, idx_rows: np.ndarray, rows: np.ndarray):
    """Oracle attention for query rows `rows` over the index lists `idx_rows`.

    Only the selected latent-KV rows travel to the host: they are gathered in
    index order and re-addressed through a per-row slot table (test plumbing; no
    arithmetic happens here)."""
    s = wl.spec
    k = idx_rows.shape[1]
    dev = wl.device
    seq_of = np.searchsorted(np_bits(wl.cu_q), rows, side="right") - 1
    idx_t = torch.from_numpy(idx_rows).to(dev).long()
    b_t = torch.from_numpy(seq_of).to(dev).long()
    valid = idx_t >= 0
    slots = wl.kv_slot_table[b_t[:, None], idx_t.clamp(min=0)].long()
    slots = torch.where(valid, slots, torch.zeros_like(slots))
    kv_rows = wl.kv[slots.reshape(-1)]
    kv_sc = None if wl.kv_scale is None else wl.kv_scale[slots.reshape(-1)]
    n = len(rows)
    table = np.arange(n * k, dtype=np.int32).reshape(n, k)
    sel = np.where(idx_rows >= 0, np.arange(k, dtype=np.int32)[None, :], -1).astype(np.int32)
    cu = np.arange(n + 1, dtype=np.int32)
    lens = np.full(n, k, dtype=np.int32)
    q_rows = wl.q[torch.from_numpy(rows).to(dev)]
    return O.sparse_mla(np_bits(q_rows), odt(q_rows), s.heads, s.d_qk, s.d_v, s.softmax_scale,
                        np_bits(kv_rows), odt(kv_rows), None if kv_sc is None else np_bits(kv_sc),
                        1, table, cu, lens, sel)


def check_logits(gpu: np.ndarray, ora: np.ndarray, pos: np.ndarray):
    for r in range(len(pos)):
        n = int(pos[r]) + 1
        g, o = gpu[r, :n].astype(np.float64), ora[r, :n].astype(np.float64)
        floor = 1e-2 * np.abs(o).max()
        tol = LOGIT_RTOL * np.maximum(np.abs(o), floor)
        bad = np.abs(g - o) > tol
        assert not bad.any(), (f"row {r}: {bad.sum()} logits out of tolerance, worst "
                               f"{np.abs(g - o)[bad].max()} at s={np.flatnonzero(bad)[:5]}")


def check_topk(gpu_idx: np.ndarray, gpu_logits: np.ndarray, ora_logits: np.ndarray,
               pos: np.ndarray, k: int):
    for r in range(len(pos)):
        n = int(pos[r]) + 1
        g = gpu_idx[r]
        m = min(k, n)
        sel = g[:m]
        assert np.all(g[m:] == -1), f"row {r}: padding"
        assert len(np.unique(sel)) == m and sel.min() >= 0 and sel.max() < n, f"row {r}: set"
        if n <= k:
            assert np.array_equal(g[:n], np.arange(n)), f"row {r}: dense fallback"
            continue
        # exact: the oracle's selection on the GPU's own scores
        exact = O.topk(gpu_logits[r:r + 1, :n], [0, 1], [n], k)[0]
        assert np.array_equal(np.sort(sel), exact), f"row {r}: top-k of identical scores differs"
        # against the oracle's scores: only near-ties at the k-th score may differ
        ref = O.topk(ora_logits[r:r + 1, :n], [0, 1], [n], k)[0]
        sk = np.sort(ora_logits[r, :n])[::-1][k - 1].astype(np.float64)
        band = TIE_RTOL * max(abs(sk), 1e-2 * np.abs(ora_logits[r, :n]).max())
        diff = np.setxor1d(sel, ref)
        far = diff[np.abs(ora_logits[r, diff].astype(np.float64) - sk) > band]
        assert far.size == 0, f"row {r}: {far.size} selections differ outside the tie band"


BF16_HALF_ULP_REL = 2.0 ** -8


def check_mla(out: np.ndarray, lse: np.ndarray, o_ref: np.ndarray, l_ref: np.ndarray, atol):
    err = np.abs(out.astype(np.float64) - o_ref.astype(np.float64))
    assert np.isfinite(out).all(), "non-finite attention output"
    tol = atol + (BF16_HALF_ULP_REL * np.abs(o_ref.astype(np.float64)) if atol >= MLA_ATOL_BF16
                  else 0.0)
    bad = err > tol
    assert not bad.any(), (f"attention error {err[bad].max()} exceeds the bound at {bad.sum()} "
                           f"elements (max abs error {err.max()})")
    lerr = np.abs(lse.astype(np.float64) - l_ref.astype(np.float64))
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    assert lerr[fin].max(initial=0) <= LSE_ATOL, f"lse max abs error {lerr[fin].max()}"


def sample_rows(T: int, n: int, seed: int = 0) -> np.ndarray:
    if T <= n:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), n - 2, replace=False)
    return np.sort(np.r_[0, mid, T - 1]).astype(np.int64)
