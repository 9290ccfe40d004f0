"""Chunked prefill of one long prompt through libdsa's C ABI.

A prompt of n_chunks x chunk_q tokens is prefilled chunk by chunk against its growing
causal prefix (chunked prefill with 8192-token chunks: "DeepSeek-V3.2-Exp DSA deployment
guide" (m.nxbn.cn), section 3.2; the context-parallelism page (lpqz.cn), section 3.1,
"--chunked-prefill-size 8192"; 128K contexts: "SGLang Day-0 support for DeepSeek-V3.2",
section "DeepSeek Sparse Attention").  Chunk c, whose queries sit at positions
[c*chunk_q, (c+1)*chunk_q):

  1. dsa_cache_store writes the chunk's new indexer-key rows (page-64 FP8 cache + scale)
     and latent-KV rows (page-1 FP8 cache + scale);
  2. dsa_indexer_topk scores every causal key of each query and keeps the top-k, in
     L2-sized row blocks (no [chunk_q][L] logits matrix);
  3. dsa_sparse_mla_prefill attends over the selected rows.

This module only sequences the calls; every step runs in the library's kernels.
"""
from __future__ import annotations

from . import dsa as L
from .workloads import INDEXER_PAGE, ChunkedWorkload


class ChunkedPrefill:
    """Buffers and calls of a whole chunked prefill on one GPU: the selection
    [n_chunks, chunk_q, k] int32, the outputs [n_chunks, chunk_q, heads, d_v] bf16 and
    lse [n_chunks, chunk_q, heads] fp32, and the indexer + top-k workspace.

    ``select_blocks="chunk"`` (the default) gives dsa_indexer_topk a workspace for a
    whole chunk's logits (8192 x 131072 fp32 = 4.3 GB at the last chunk), so each
    chunk's indexer and top-k run as one launch each; ``"l2"`` gives it the minimum,
    so it works in L2-sized row blocks (about 80 MB of logits, hundreds of launches)."""

    def __init__(self, cw: ChunkedWorkload, select_blocks: str = "chunk"):
        import torch
        s = cw.spec
        self.cw, self.s = cw, s
        dev = cw.device
        C, Q = s.n_chunks, s.chunk_q
        self.batches = [L.Batch(cw.cu_q, cw.seq_lens[c:c + 1], Q, Q * (c + 1)) for c in range(C)]
        self.kc = L.PagedCache(cw.k_pages, cw.k_block_table, INDEXER_PAGE, cw.k_scale)
        self.kvc = L.PagedCache(cw.kv, cw.kv_slot_table, 1, cw.kv_scale)
        self.idx = torch.empty(C, Q, s.topk, dtype=torch.int32, device=dev)
        self.out = torch.empty(C, Q, s.heads, s.d_v, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(C, Q, s.heads, device=dev)
        if select_blocks not in ("chunk", "l2"):
            raise ValueError("select_blocks must be 'chunk' or 'l2'")
        n = max(L.dsa_indexer_topk_workspace_size(b) for b in self.batches)
        if select_blocks == "chunk":
            n = max(n, Q * ((Q * C + 63) // 64 * 64) * 4)
        self.ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)

    def rows(self, c: int):
        Q = self.s.chunk_q
        return slice(c * Q, (c + 1) * Q)

    # the three calls of chunk c, on caller-chosen input / output tensors
    def store(self, c, k_rows, kv_rows, k_slots, kv_slots, stream=None):
        cw = self.cw
        L.dsa_cache_store(k_rows, k_slots, cw.k_pages, cw.k_scale, stream=stream)
        L.dsa_cache_store(kv_rows, kv_slots, cw.kv, cw.kv_scale, stream=stream)

    def select(self, c, q_idx, w, idx, stream=None):
        L.dsa_indexer_topk(q_idx, None, w, self.kc, self.batches[c], self.s.topk, idx,
                           workspace=self.ws, stream=stream)

    def attend(self, c, q, idx, out, lse, stream=None):
        s = self.s
        L.dsa_sparse_mla_prefill(q, self.kvc, self.batches[c], idx, s.d_v, s.softmax_scale,
                                 out, lse, stream=stream)

    # resident inputs and outputs
    def chunk(self, c: int):
        cw, r = self.cw, self.rows(c)
        self.store(c, cw.k_new[r], cw.kv_new[r], cw.k_slots[r], cw.kv_slots[r])
        self.select(c, cw.q_idx[c], cw.w[c], self.idx[c])
        self.attend(c, cw.q[c], self.idx[c], self.out[c], self.lse[c])

    def step(self):
        """The whole prompt, chunk after chunk."""
        for c in range(self.s.n_chunks):
            self.chunk(c)

    def stages(self):
        """The same calls grouped by stage over all chunks (for per-stage timing; every
        chunk's rows are stored before any chunk is scored, so causality holds)."""
        cw, C = self.cw, self.s.n_chunks

        def store_all():
            for c in range(C):
                r = self.rows(c)
                self.store(c, cw.k_new[r], cw.kv_new[r], cw.k_slots[r], cw.kv_slots[r])

        def select_all():
            for c in range(C):
                self.select(c, cw.q_idx[c], cw.w[c], self.idx[c])

        def attend_all():
            for c in range(C):
                self.attend(c, cw.q[c], self.idx[c], self.out[c], self.lse[c])

        return [store_all, select_all, attend_all]

    def launches_per_step(self) -> int:
        """Kernel launches of one step: two stores, the indexer and top-k once per row
        block, and the attention, per chunk."""
        n = 0
        ws = self.ws.numel()
        for b in self.batches:
            ld = (b.max_seq_len + 63) // 64 * 64
            rows = _block_rows(b.total_q, ld, ws)
            n += 2 + 2 * ((b.total_q + rows - 1) // rows) + 1
        return n


def _block_rows(total_q: int, ld: int, ws_bytes: int = 0) -> int:
    """Rows per block of dsa_indexer_topk for a workspace of ws_bytes (the library's
    rule, restated for counting)."""
    budget = max(80 << 20, ws_bytes) // (ld * 4)
    if budget >= total_q:
        return total_q
    if budget >= 148:
        rows = 148
        while rows * 2 <= budget:
            rows *= 2
    else:
        rows = budget & ~3
    return max(4, min(rows, total_q))
