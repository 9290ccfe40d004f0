"""GPU parity of libdsa against the CPU oracle, through the C ABI.

Each workload shape runs at full size in the launch configuration the benchmark
uses; the oracle recomputes sampled query rows (all rows where it finishes in
seconds).  Tolerances are stated in tests/_helpers.py.
"""
import math

import numpy as np
import pytest
import torch

import long_context_sparse_fp8_b200 as L
from long_context_sparse_fp8_b200 import chunked as CH
from long_context_sparse_fp8_b200 import workloads as W
from oracle import oracle as O

import _helpers as H

pytestmark = pytest.mark.gpu

_CACHE = {}


def _wl(key, spec_fn):
    if key not in _CACHE:
        _CACHE.clear()
        torch.cuda.empty_cache()
        _CACHE[key] = W.make(spec_fn(), device="cuda")
    return _CACHE[key]


def _pipeline(wl, rows, decode=False, atol=H.MLA_ATOL_BF16):
    assert L.dsa_device_check() == 0
    logits = H.run_indexer(wl)
    idx = H.run_topk(wl, logits)
    out, lse = H.run_mla(wl, idx, decode=decode)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    pos = H.positions(wl)[rows]
    rows_t = torch.from_numpy(rows).cuda()
    g_logits = logits[rows_t].cpu().numpy()
    o_logits = H.oracle_logits(wl, rows)
    H.check_logits(g_logits, o_logits, pos)
    g_idx = idx[rows_t].cpu().numpy()
    H.check_topk(g_idx, g_logits, o_logits, pos, wl.spec.topk)
    o_ref, l_ref = H.oracle_mla(wl, g_idx, rows)
    H.check_mla(out[rows_t].float().cpu().numpy(), lse[rows_t].cpu().numpy(), o_ref, l_ref, atol)
    return logits, idx, out, lse


def test_tiny_prefill_all_rows():
    wl = W.make(W.tiny_prefill(), device="cuda")
    _pipeline(wl, np.arange(wl.spec.total_q), atol=H.MLA_ATOL_F32)


def test_decode_b32_ctx8192():
    wl = _wl("c2", W.decode_b32_8k)
    _pipeline(wl, np.arange(32), decode=True)


def test_fused_decode_matches_separate_calls():
    wl = _wl("c2", W.decode_b32_8k)
    s = wl.spec
    batch, kc, kv = H.lib_args(wl)
    logits = H.run_indexer(wl)
    idx = H.run_topk(wl, logits)
    out, lse = H.run_mla(wl, idx, decode=True)
    n = L.dsa_decode_workspace_size(batch, s.topk, s.heads, s.d_v)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    idx2 = torch.empty_like(idx)
    L.dsa_decode(wl.q_idx, None, wl.w, kc, s.topk, wl.q, kv, batch, s.d_v, s.softmax_scale, out2,
                 lse2, idx2, ws)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    assert torch.equal(idx, idx2)          # top-k output is deterministic
    assert torch.equal(out, out2)
    assert torch.equal(lse, lse2)


@pytest.mark.parametrize("nq", [2, 3, 4])
def test_multi_query_decode(nq):
    """Decode with nq query tokens per sequence (a multi-token-prediction verify step):
    the fused call against the oracle on sampled rows, each later token of a sequence
    seeing one more key."""
    wl = _wl(f"mtp{nq}", lambda: W.decode_mtp_b32_8k(nq))
    s = wl.spec
    batch, kc, kv = H.lib_args(wl)
    n = L.dsa_decode_workspace_size(batch, s.topk, s.heads, s.d_v)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.empty(s.total_q, s.heads, s.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(s.total_q, s.heads, device="cuda")
    idx = torch.empty(s.total_q, s.topk, dtype=torch.int32, device="cuda")
    L.dsa_decode(wl.q_idx, None, wl.w, kc, s.topk, wl.q, kv, batch, s.d_v, s.softmax_scale, out,
                 lse, idx, ws)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    rows = np.unique(np.concatenate([H.sample_rows(s.total_q, 10, seed=20 + nq),
                                     np.arange(nq)]))           # all tokens of sequence 0
    pos = H.positions(wl)[rows]
    o_logits = H.oracle_logits(wl, rows)
    g_idx = idx.cpu().numpy()[rows]
    # the fused call keeps its logits in the workspace; the stand-alone indexer call
    # (same kernel) gives the scores its selection must be exact on
    g_logits = H.run_indexer(wl).cpu().numpy()[rows]
    H.check_logits(g_logits, o_logits, pos)
    H.check_topk(g_idx, g_logits, o_logits, pos, s.topk)
    o_ref, l_ref = H.oracle_mla(wl, g_idx, rows)
    H.check_mla(out.float().cpu().numpy()[rows], lse.cpu().numpy()[rows], o_ref, l_ref,
                H.MLA_ATOL_BF16)
    _pipeline(wl, rows, decode=True)


def test_prefill_32k_heavy_hitters():
    wl = _wl("c3", W.prefill_32k)
    _pipeline(wl, H.sample_rows(wl.spec.total_q, 64, seed=3))


def test_decode_b64_paged_fp8_kv():
    wl = _wl("c4", W.decode_b64_128k)
    _pipeline(wl, H.sample_rows(64, 8, seed=4), decode=True)


def test_chunked_prefill_128k_whole_prompt():
    """The whole 131072-token prefill in 16 chunks of 8192, run as the benchmark runs it
    (per chunk: dsa_cache_store of the chunk's key and latent-KV rows, dsa_indexer_topk,
    dsa_sparse_mla_prefill).  The caches it wrote must equal the oracle's cache_store of
    the same rows byte for byte; on chunks 0, 7, 11 and 15, 64 rows each (first, last and
    62 drawn), the indexer logits, the selection and the attention output are checked
    against the oracle computed over the oracle's own caches."""
    _CACHE.clear()
    torch.cuda.empty_cache()
    cw = W.make_chunked(W.ChunkedSpec(), device="cuda")
    s = cw.spec
    cp = CH.ChunkedPrefill(cw)
    cp.step()
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    slots = np.arange(s.seq_len, dtype=np.int64)
    kd, ks = O.cache_store(H.np_bits(cw.k_new), O.BF16, slots,
                           np.zeros((s.seq_len, s.idx_dim), np.uint8), O.E4M3,
                           np.zeros(s.seq_len, np.float32))
    vd, vs = O.cache_store(H.np_bits(cw.kv_new), O.BF16, slots,
                           np.zeros((s.seq_len, s.d_qk), np.uint8), O.E4M3,
                           np.zeros(s.seq_len, np.float32))
    assert np.array_equal(H.np_bits(cw.k_pages).reshape(s.seq_len, -1), kd)
    assert np.array_equal(H.np_bits(cw.kv), vd)
    assert np.array_equal(H.np_bits(cw.k_scale).reshape(-1).view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(H.np_bits(cw.kv_scale).view(np.uint32), vs.view(np.uint32))
    caches = (torch.from_numpy(kd).cuda().view(W.FP8).reshape(-1, W.INDEXER_PAGE, s.idx_dim),
              torch.from_numpy(ks).cuda().reshape(-1, W.INDEXER_PAGE),
              torch.from_numpy(vd).cuda().view(W.FP8), torch.from_numpy(vs).cuda())
    for c in (0, 7, 11, 15):
        wl = W.chunk_view(cw, c, *caches)
        rows = H.sample_rows(s.chunk_q, 64, seed=50 + c)
        pos = H.positions(wl)[rows]
        # the chunk's logits from the stand-alone indexer call (the same kernel and row
        # grouping as the row blocks of dsa_indexer_topk): the selection must be exact on them
        logits = H.run_indexer(W.chunk_view(cw, c))
        rows_t = torch.from_numpy(rows).cuda()
        g_logits = logits[rows_t].cpu().numpy()
        del logits
        o_logits = H.oracle_logits(wl, rows)
        H.check_logits(g_logits, o_logits, pos)
        g_idx = cp.idx[c][rows_t].cpu().numpy()
        H.check_topk(g_idx, g_logits, o_logits, pos, s.topk)
        o_ref, l_ref = H.oracle_mla(wl, g_idx, rows)
        H.check_mla(cp.out[c][rows_t].float().cpu().numpy(), cp.lse[c][rows_t].cpu().numpy(),
                    o_ref, l_ref, H.MLA_ATOL_BF16)
    del cp, cw
    torch.cuda.empty_cache()


@pytest.mark.parametrize("kv_fp8,permute", [(False, False), (True, True)])
def test_ragged_batch_edge_cases(kv_fp8, permute):
    """Lengths around page edges, L < k, a sequence with no queries, many queries."""
    spec = W.Spec(name="ragged", seq_lens=[1, 63, 64, 65, 200, 2100, 3000, 2049],
                  nq=[1, 5, 64, 2, 0, 7, 30, 3], topk=2048, kv_fp8=kv_fp8,
                  permute_tables=permute, seed=77)
    wl = W.make(spec, device="cuda")
    _pipeline(wl, np.arange(spec.total_q))
    _pipeline(wl, np.arange(spec.total_q), decode=True)


def test_small_k_and_fp32_mla_split():
    spec = W.tiny_prefill(seed=99)
    spec.seq_lens, spec.nq, spec.topk = [300, 129], [40, 129], 16
    wl = W.make(spec, device="cuda")
    _pipeline(wl, np.arange(spec.total_q), atol=H.MLA_ATOL_F32)
    _pipeline(wl, np.arange(spec.total_q), decode=True, atol=H.MLA_ATOL_F32)


@pytest.mark.parametrize("n,k,kind", [(5000, 2048, "equal"), (5000, 2048, "three"),
                                      (2049, 2048, "zeros"), (70000, 2048, "three"),
                                      (70000, 2048, "normal"), (2048, 2048, "normal"),
                                      (100000, 4096, "equal"), (50000, 2048, "coarse"),
                                      (20000, 2048, "normal"), (9000, 100, "coarse"),
                                      (300000, 2048, "normal"), (300000, 2048, "three"),
                                      (100000, 65536, "normal"), (65536, 65536, "coarse")])
def test_topk_ties_and_long_rows(n, k, kind):
    g = torch.Generator(device="cuda").manual_seed(n + k)
    if kind == "equal":
        row = torch.full((1, n), 1.5, device="cuda")
    elif kind == "three":
        row = torch.randint(0, 3, (1, n), generator=g, device="cuda").float()
    elif kind == "zeros":  # +0.0 and -0.0 compare equal
        row = torch.zeros(1, n, device="cuda")
        row[0, ::2] = -0.0
    elif kind == "coarse":  # many exact ties around the k-th score
        row = torch.round(torch.randn(1, n, generator=g, device="cuda") * 50) / 50
    else:
        row = torch.randn(1, n, generator=g, device="cuda")
    ld = (n + 3) // 4 * 4
    logits = torch.full((1, ld), float("nan"), device="cuda")
    logits[:, :n] = row
    batch = L.Batch(torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
                    torch.tensor([n], dtype=torch.int32, device="cuda"), 1, n)
    idx = torch.empty(1, k, dtype=torch.int32, device="cuda")
    L.dsa_topk(logits, batch, k, idx)
    got = idx.cpu().numpy()
    H.check_topk(got, logits.cpu().numpy(), logits.cpu().numpy(), np.array([n - 1]), k)
    if kind == "equal":
        assert np.array_equal(np.sort(got[0]), np.arange(k))


def test_topk_candidates_concentrated_in_one_warp():
    # The keys of the k-th key's top-bit bin all sit in 32-key groups that one warp of
    # the top-k CTA sweeps (every 32nd group), so that warp's candidate segment
    # overflows and the row must take the whole-row fallback -- same result required.
    n, k = 60000, 2048
    pos = np.arange(n)
    row = np.zeros(n, dtype=np.float32)
    mine = np.flatnonzero((pos // 32) % 32 == 0)[:900]         # 900 candidates, one warp
    row[mine] = 5.0 + (np.arange(len(mine)) % 97) * 1e-3        # same 11-bit bin, many ties
    top = np.setdiff1d(pos, mine)[::37][:1500]                  # 1500 keys above that bin
    row[top] = 10.0
    ld = (n + 3) // 4 * 4
    logits = torch.full((1, ld), float("nan"), device="cuda")
    logits[0, :n] = torch.from_numpy(row).cuda()
    batch = L.Batch(torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
                    torch.tensor([n], dtype=torch.int32, device="cuda"), 1, n)
    idx = torch.empty(1, k, dtype=torch.int32, device="cuda")
    L.dsa_topk(logits, batch, k, idx)
    got = idx.cpu().numpy()
    H.check_topk(got, logits.cpu().numpy(), logits.cpu().numpy(), np.array([n - 1]), k)


@pytest.mark.parametrize("case", ["few_reach_threshold", "one_warp_overflows", "all_reach"])
def test_topk_sampled_threshold_falls_back(case):
    """Rows of >= 24k keys first try a threshold taken from 2048 evenly spaced keys.  Rows
    built against it must still get the exact selection: (a) only the sampled positions
    hold large scores, so fewer than k keys reach the sampled threshold; (b) the keys
    that reach it all sit in the 128-key blocks one warp reads, overflowing its
    candidate segment; (c) every key reaches it (a constant row)."""
    n, k = 60000, 2048
    pos = np.arange(n)
    g = np.random.default_rng(7)
    row = g.standard_normal(n).astype(np.float32)
    if case == "few_reach_threshold":
        samp = (np.arange(2048) * n) // 2048                # the sampled positions
        row[samp] = 100.0 + np.arange(2048, dtype=np.float32)
    elif case == "one_warp_overflows":
        mine = np.flatnonzero((pos // 128) % 32 == 0)[:3000]
        row[mine] = 50.0 + g.standard_normal(len(mine)).astype(np.float32)
    else:
        row[:] = 0.25
    ld = (n + 3) // 4 * 4
    logits = torch.full((1, ld), float("nan"), device="cuda")
    logits[0, :n] = torch.from_numpy(row).cuda()
    batch = L.Batch(torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
                    torch.tensor([n], dtype=torch.int32, device="cuda"), 1, n)
    idx = torch.empty(1, k, dtype=torch.int32, device="cuda")
    L.dsa_topk(logits, batch, k, idx)
    got = idx.cpu().numpy()
    assert L.dsa_device_check() == 0
    H.check_topk(got, logits.cpu().numpy(), logits.cpu().numpy(), np.array([n - 1]), k)
    if case == "few_reach_threshold":
        assert np.array_equal(got[0], (np.arange(2048) * n) // 2048)
    if case == "all_reach":
        assert np.array_equal(got[0], np.arange(k))


@pytest.mark.parametrize("kind", ["normal", "coarse", "three"])
def test_topk_cluster_split_matches_one_cta_per_row(kind):
    """Short batches of long rows split each row over a cluster of 8, 4 or 2 CTAs;
    larger batches give each row one CTA.  The same rows must get the same lists
    either way (ragged lengths, so some clusters hold rows far shorter than the
    longest)."""
    n, k, T = 40000, 2048, 200
    g = torch.Generator(device="cuda").manual_seed(99)
    x = torch.randn(T, n, generator=g, device="cuda")
    if kind == "coarse":
        x = torch.round(x * 20) / 20
    elif kind == "three":
        x = torch.randint(0, 3, (T, n), generator=g, device="cuda").float()
    lens = torch.randint(3000, n + 1, (T,), generator=g, device="cuda").to(torch.int32)
    lens[0] = n
    logits = x.contiguous()
    def run(rows):
        cu = torch.arange(rows + 1, dtype=torch.int32, device="cuda")
        b = L.Batch(cu, lens[:rows].contiguous(), rows, n)
        idx = torch.empty(rows, k, dtype=torch.int32, device="cuda")
        L.dsa_topk(logits[:rows], b, k, idx)
        torch.cuda.synchronize()
        return idx.cpu().numpy()
    full = run(T)                                  # one CTA per row
    for rows in (16, 36, 72):                      # clusters of 8, 4, 2
        part = run(rows)
        assert np.array_equal(part, full[:rows]), rows
    assert L.dsa_device_check() == 0
    pos = lens.cpu().numpy() - 1
    lg = logits.cpu().numpy()
    sel = np.array([0, 5, 71])
    H.check_topk(full[sel], lg[sel], lg[sel], pos[sel], k)


@pytest.mark.parametrize("which", ["prefill_32k", "fp32_blocks", "ragged"])
def test_indexer_topk_blocks_match_separate_calls(which):
    """dsa_indexer_topk (L2-sized row blocks, no full logits matrix) selects exactly what
    dsa_indexer_logits + dsa_topk select: 14 blocks of up to 592 rows on the 32K prefill
    (FP8 tensor-core indexer), 4 blocks on an fp32 case (CUDA-core indexer); and so it
    does with larger workspaces (larger blocks, up to the whole batch in one)."""
    if which == "prefill_32k":
        wl = _wl("c3", W.prefill_32k)
    elif which == "ragged":
        spec = W.Spec(name="ragged", seq_lens=[1, 63, 64, 65, 200, 2100, 3000, 2049],
                      nq=[1, 5, 64, 2, 0, 7, 30, 3], topk=2048, seed=77)
        wl = W.make(spec, device="cuda")
    else:
        spec = W.Spec(name="blocks_f32", seq_lens=[40000, 30000], nq=[700, 300], topk=64,
                      idx_heads=4, idx_dim=32, idx_fp8=False, w_std=0.5, heads=2, d_qk=80,
                      d_v=64, mla_dtype="f32", softmax_scale=1.0 / math.sqrt(80.0), seed=31)
        wl = W.make(spec, device="cuda")
    s = wl.spec
    batch, kc, _ = H.lib_args(wl)
    logits = H.run_indexer(wl)
    idx = H.run_topk(wl, logits)
    ws_bytes = L.dsa_indexer_topk_workspace_size(batch)
    ld = (s.max_seq_len + 63) // 64 * 64
    assert ws_bytes < s.total_q * ld * 4 or s.total_q * ld * 4 <= 80 << 20
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    idx2 = torch.full_like(idx, -7)
    L.dsa_indexer_topk(wl.q_idx, None, wl.w, kc, batch, s.topk, idx2, workspace=ws)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    assert torch.equal(idx, idx2)
    # larger workspaces take larger blocks: 148 x 2^m rows, then the whole batch at once
    for bytes_ in (2 * 148 * ld * 4 + 100, s.total_q * ld * 4):
        if bytes_ <= ws_bytes:
            continue
        ws_big = torch.empty(bytes_, dtype=torch.uint8, device="cuda")
        idx3 = torch.full_like(idx, -7)
        L.dsa_indexer_topk(wl.q_idx, None, wl.w, kc, batch, s.topk, idx3, workspace=ws_big)
        torch.cuda.synchronize()
        assert L.dsa_device_check() == 0
        assert torch.equal(idx, idx3), bytes_
        del ws_big
    rows = H.sample_rows(s.total_q, 6, seed=41)
    pos = H.positions(wl)[rows]
    g = logits.cpu().numpy()[rows]
    H.check_topk(idx2.cpu().numpy()[rows], g, H.oracle_logits(wl, rows), pos, s.topk)


def test_device_check_reports_bad_index_and_page():
    spec = W.Spec(name="chk", seq_lens=[300], nq=[4], topk=64, seed=5)
    wl = W.make(spec, device="cuda")
    assert L.dsa_device_check() == 0
    logits = H.run_indexer(wl)
    idx = H.run_topk(wl, logits)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    bad = idx.clone()
    bad[0, 3] = 299  # row 0 sits at position 296
    out, lse = H.run_mla(wl, bad)
    assert L.dsa_device_check(reset=True) == 2  # DSA_CHECK_BAD_INDEX
    assert torch.isfinite(out.float()).all()
    assert L.dsa_device_check() == 0
    wl.k_block_table[0, 2] = 10_000  # outside the page pool
    H.run_indexer(wl)
    assert L.dsa_device_check(reset=True) == 1  # DSA_CHECK_BAD_PAGE


def test_empty_batch_is_a_no_op():
    spec = W.Spec(name="empty", seq_lens=[10], nq=[0], topk=8, seed=1)
    wl = W.make(spec, device="cuda")
    batch, kc, kv = H.lib_args(wl)
    logits = torch.full((1, 64), 3.0, device="cuda")
    L.dsa_indexer_logits(wl.q_idx, None, wl.w, kc, batch, logits)
    idx = torch.full((1, 8), 5, dtype=torch.int32, device="cuda")
    L.dsa_topk(logits, batch, 8, idx)
    torch.cuda.synchronize()
    assert L.dsa_device_check() == 0
    assert torch.all(logits == 3.0) and torch.all(idx == 5)


def test_back_to_back_fused_decodes_share_a_workspace():
    """Two dsa_decode calls queued back to back on one stream, the second on a different
    batch, both keeping their selection in the same workspace: each kernel of the
    second call waits for the kernel before it before writing anything, so the second
    call's top-k cannot overwrite the selection the first call's attention still
    reads.  40 rows (one split, no merge kernel), some shorter than k."""
    lens_a = [1500, 3000, 900, 4100, 2047, 2048, 2049, 5000] * 5
    lens_b = [4000, 1200, 2600, 300, 5000, 2100, 64, 3500] * 5
    wls = [W.make(W.Spec(name=f"b2b{i}", seq_lens=lens, nq=[1] * len(lens), topk=2048,
                         seed=300 + i), device="cuda")
           for i, lens in enumerate((lens_a, lens_b))]
    s = wls[0].spec
    ref = []
    for wl in wls:
        idx = H.run_topk(wl, H.run_indexer(wl))
        out, lse = H.run_mla(wl, idx, decode=True)
        ref.append((idx, out, lse))
    torch.cuda.synchronize()
    n = max(L.dsa_decode_workspace_size(H.lib_args(wl)[0], s.topk, s.heads, s.d_v) for wl in wls)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    for rep in range(3):
        got = []
        for wl in wls:
            batch, kc, kv = H.lib_args(wl)
            out = torch.empty(s.total_q, s.heads, s.d_v, dtype=torch.bfloat16, device="cuda")
            lse = torch.empty(s.total_q, s.heads, device="cuda")
            L.dsa_decode(wl.q_idx, None, wl.w, kc, s.topk, wl.q, kv, batch, s.d_v,
                         s.softmax_scale, out, lse, None, ws)
            got.append((out, lse))
        torch.cuda.synchronize()
        assert L.dsa_device_check() == 0
        for (_, r_out, r_lse), (g_out, g_lse) in zip(ref, got):
            assert torch.equal(r_out, g_out), rep
            assert torch.equal(r_lse, g_lse), rep


@pytest.mark.parametrize("where", ["kv", "q", "q_fp8_cache"])
def test_fp16_range_is_reported(where):
    """The tensor-core attention computes on fp16 operands: a bf16 latent-KV row or query
    (next to a bf16 or an fp8 cache) with entries beyond +-65504 cannot be represented
    there, and the call must say so (DSA_CHECK_FP16_RANGE) instead of returning silently
    saturated results.  Rows of ordinary magnitude in the same call are still exact."""
    spec = W.Spec(name="range", seq_lens=[3000, 2500], nq=[3, 2], topk=2048,
                  kv_fp8=(where == "q_fp8_cache"), seed=91)
    wl = W.make(spec, device="cuda")
    if where == "kv":
        wl.kv[17, :8] = 1.0e5                      # slot 17 = position 17 of sequence 0
        wl.kv[18, 100] = -2.0e5
    else:
        wl.q[1, 5, 7] = 1.0e5
    idx = torch.arange(spec.topk, dtype=torch.int32, device="cuda").repeat(spec.total_q, 1)
    pos = torch.from_numpy(H.positions(wl)).cuda()
    idx = torch.where(idx <= pos[:, None], idx, torch.full_like(idx, -1))
    assert L.dsa_device_check() == 0
    out, lse = H.run_mla(wl, idx)
    torch.cuda.synchronize()
    assert L.dsa_device_check(reset=True) == 5     # DSA_CHECK_FP16_RANGE
    assert L.dsa_device_check() == 0
    # the rows of sequence 1 see neither the large KV rows nor the large query value
    rows = np.array([3, 4])
    o_ref, l_ref = H.oracle_mla(wl, idx.cpu().numpy()[rows], rows)
    H.check_mla(out[3:5].float().cpu().numpy(), lse[3:5].cpu().numpy(), o_ref, l_ref,
                H.MLA_ATOL_BF16)
