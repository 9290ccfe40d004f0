"""Seeded synthetic DSA workloads shared by the library's tests, smoke check and bench.

This module only draws random tensors and lays them out in the cache formats the
library reads; it holds none of the DSA arithmetic (no scoring, selection or
attention).  Both the CUDA path and the CPU oracle consume exactly the tensors
made here.

Cache formats (from "SGLang Day-0 support for DeepSeek-V3.2", section "DeepSeek
Sparse Attention": the indexer key & key_scale cache uses page size 64, the
token-level sparse operator page size 1; fp8_e4m3 KV from "DeepSeek-V3.2-Exp DSA
deployment guide", section 3.1):

* indexer keys   ``k_pages [num_pages, 64, d_I]`` (fp8 e4m3 or fp32) with
  ``k_scale [num_pages, 64]`` fp32 (one positive scale per token, amax/448), and
  ``k_block_table [B, max_pages]`` int32 (logical page -> physical page, -1 unused);
* latent KV      ``kv [num_slots, 576]`` (bf16, or fp8 e4m3 with ``kv_scale
  [num_slots]`` fp32), page size 1, ``kv_slot_table [B, max_len]`` int32;
* queries of sequence b are its last ``nq_b`` tokens; ``cu_q [B+1]`` int32.

Value recipe: N(0,1) draws; fp8 tensors are quantised with a per-token scale
amax/448 (values clamped to the e4m3 range before the cast); indexer queries are
N(0,1) cast straight to e4m3; indexer head weights w ~ N(0,1)/sqrt(H_I)-style
(as each workload states); optional "heavy hitters" multiply the indexer key and
the latent-KV row of a seeded 1% of positions by 4 before quantisation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

FP8 = torch.float8_e4m3fn
FP8_MAX = 448.0
INDEXER_PAGE = 64


@dataclass
class Spec:
    """Shape and value recipe of one synthetic DSA workload."""
    name: str
    seq_lens: List[int]
    nq: List[int]
    topk: int
    # indexer
    idx_heads: int = 64
    idx_dim: int = 128
    idx_fp8: bool = True
    w_std: float = 1.0 / 8.0
    # sparse MLA
    heads: int = 128
    d_qk: int = 576
    d_v: int = 512
    mla_dtype: str = "bf16"        # "f32" | "bf16"  (q and bf16/f32 KV)
    kv_fp8: bool = False
    softmax_scale: float = 1.0 / math.sqrt(192.0)
    # layout / values
    permute_tables: bool = False
    heavy_frac: float = 0.0
    heavy_mult: float = 4.0
    seed: int = 1234

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def total_q(self) -> int:
        return int(sum(self.nq))

    @property
    def max_seq_len(self) -> int:
        return int(max(self.seq_lens))


@dataclass
class Workload:
    spec: Spec
    cu_q: torch.Tensor            # [B+1] int32
    seq_lens: torch.Tensor        # [B] int32
    # indexer
    q_idx: torch.Tensor           # [T, H_I, d_I] fp8 or fp32
    w: torch.Tensor               # [T, H_I] fp32
    k_pages: torch.Tensor         # [P, 64, d_I] fp8 or fp32
    k_scale: Optional[torch.Tensor]   # [P, 64] fp32 or None
    k_block_table: torch.Tensor   # [B, max_pages] int32
    # MLA
    q: torch.Tensor               # [T, heads, d_qk] bf16 or fp32
    kv: torch.Tensor              # [S, d_qk] bf16 / fp32 / fp8
    kv_scale: Optional[torch.Tensor]  # [S] fp32 or None
    kv_slot_table: torch.Tensor   # [B, max_len] int32
    extra: dict = field(default_factory=dict)

    @property
    def device(self):
        return self.q.device


def _quant_rows_fp8(x: torch.Tensor):
    """Per-row fp8 e4m3 codes and fp32 scale amax/448 (scale 1 for all-zero rows)."""
    amax = x.abs().amax(dim=-1).float()
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    codes = (x.float() / scale.unsqueeze(-1)).clamp_(-FP8_MAX, FP8_MAX).to(FP8)
    return codes, scale


def _tables(spec: Spec, units_per_seq: List[int], gen_cpu: torch.Generator, width: int):
    """Logical->physical tables; identity-by-sequence, or one seeded permutation."""
    total = int(sum(units_per_seq))
    if spec.permute_tables:
        phys = torch.randperm(total, generator=gen_cpu).to(torch.int32)
    else:
        phys = torch.arange(total, dtype=torch.int32)
    table = torch.full((spec.num_seqs, width), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(units_per_seq):
        table[b, :n] = phys[off:off + n]
        off += n
    return table, total


def make(spec: Spec, device="cpu") -> Workload:
    """Draw the workload ``spec`` on ``device`` (seeded; cuda draws use torch's Philox)."""
    device = torch.device(device)
    g_cpu = torch.Generator().manual_seed(spec.seed)
    g = torch.Generator(device=device).manual_seed(spec.seed + 1)
    B, T = spec.num_seqs, spec.total_q
    seq_lens = torch.tensor(spec.seq_lens, dtype=torch.int32)
    cu_q = torch.zeros(B + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(torch.tensor(spec.nq, dtype=torch.int64), 0).to(torch.int32)
    for b in range(B):
        if not (0 <= spec.nq[b] <= spec.seq_lens[b]):
            raise ValueError("each sequence needs 0 <= nq <= L")

    # --- indexer key cache (page 64) ---
    pages_per_seq = [(L + INDEXER_PAGE - 1) // INDEXER_PAGE for L in spec.seq_lens]
    k_bt, n_pages = _tables(spec, pages_per_seq, g_cpu, max(pages_per_seq))
    # --- latent KV cache (page 1) ---
    kv_st, n_slots = _tables(spec, list(spec.seq_lens), g_cpu, spec.max_seq_len)

    # heavy hitters: a seeded 1% of each sequence's positions
    heavy = []
    for L in spec.seq_lens:
        n_h = int(round(spec.heavy_frac * L))
        heavy.append(torch.randperm(L, generator=g_cpu)[:n_h] if n_h else None)

    dI, HI = spec.idx_dim, spec.idx_heads
    k_pages = torch.zeros(n_pages, INDEXER_PAGE, dI, dtype=FP8 if spec.idx_fp8 else torch.float32,
                          device=device)
    k_scale = torch.ones(n_pages, INDEXER_PAGE, dtype=torch.float32, device=device) \
        if spec.idx_fp8 else None
    kv_dt = FP8 if spec.kv_fp8 else (torch.bfloat16 if spec.mla_dtype == "bf16" else torch.float32)
    kv = torch.zeros(n_slots, spec.d_qk, dtype=kv_dt, device=device)
    kv_scale = torch.ones(n_slots, dtype=torch.float32, device=device) if spec.kv_fp8 else None

    k_bt_dev = k_bt.to(device)
    kv_st_dev = kv_st.to(device)
    CH = 16384  # draw in chunks to bound temporary memory
    for b, L in enumerate(spec.seq_lens):
        for s0 in range(0, L, CH):
            s1 = min(L, s0 + CH)
            pos = torch.arange(s0, s1, device=device)
            kk = torch.randn(s1 - s0, dI, generator=g, device=device)
            vv = torch.randn(s1 - s0, spec.d_qk, generator=g, device=device)
            if heavy[b] is not None:
                hb = heavy[b].to(device)
                sel = hb[(hb >= s0) & (hb < s1)] - s0
                kk[sel] *= spec.heavy_mult
                vv[sel] *= spec.heavy_mult
            page = k_bt_dev[b, pos // INDEXER_PAGE].long()
            row = pos % INDEXER_PAGE
            if spec.idx_fp8:
                codes, sc = _quant_rows_fp8(kk)
                k_pages[page, row] = codes
                k_scale[page, row] = sc
            else:
                k_pages[page, row] = kk
            slot = kv_st_dev[b, pos].long()
            if spec.kv_fp8:
                codes, sc = _quant_rows_fp8(vv)
                kv[slot] = codes
                kv_scale[slot] = sc
            else:
                kv[slot] = vv.to(kv_dt)

    qi = torch.randn(T, HI, dI, generator=g, device=device)
    q_idx = qi.clamp(-FP8_MAX, FP8_MAX).to(FP8) if spec.idx_fp8 else qi
    w = torch.randn(T, HI, generator=g, device=device) * spec.w_std
    q_dt = torch.bfloat16 if spec.mla_dtype == "bf16" else torch.float32
    q = torch.randn(T, spec.heads, spec.d_qk, generator=g, device=device).to(q_dt)

    return Workload(spec=spec, cu_q=cu_q.to(device), seq_lens=seq_lens.to(device), q_idx=q_idx,
                    w=w, k_pages=k_pages, k_scale=k_scale, k_block_table=k_bt_dev, q=q, kv=kv,
                    kv_scale=kv_scale, kv_slot_table=kv_st_dev,
                    extra={"heavy": heavy})


# ----------------------------------------------------------------------------------------
# The five workload shapes (sizes as stated for each; seeds 1234 + id).
# ----------------------------------------------------------------------------------------

def tiny_prefill(seed: int = 1235) -> Spec:
    """1 sequence L=256, all 256 queries causal; indexer 4 heads x 32 fp32, w ~ N(0,1)/2;
    top-k 64; MLA 2 heads, 64 latent + 16 rope, d_v 64, fp32, scale 1/sqrt(80)."""
    return Spec(name="tiny_prefill_L256", seq_lens=[256], nq=[256], topk=64, idx_heads=4,
                idx_dim=32, idx_fp8=False, w_std=0.5, heads=2, d_qk=80, d_v=64,
                mla_dtype="f32", softmax_scale=1.0 / math.sqrt(80.0), seed=seed)


def decode_b32_8k(seed: int = 1236) -> Spec:
    """Decode, 32 sequences x 8192 context, 1 query each; FP8 indexer 64x128, top-k 2048;
    128-head MLA over bf16 576-d latent KV."""
    return Spec(name="decode_b32_ctx8192", seq_lens=[8192] * 32, nq=[1] * 32, topk=2048,
                seed=seed)


def decode_mtp_b32_8k(nq: int = 2, seed: int = 1241) -> Spec:
    """Multi-query decode (a verify step of multi-token prediction): 32 sequences x 8192
    context, ``nq`` query tokens each (the last nq positions); otherwise as the
    32 x 8192 decode."""
    return Spec(name=f"decode_mtp{nq}_b32_ctx8192", seq_lens=[8192] * 32, nq=[nq] * 32,
                topk=2048, seed=seed)


def prefill_32k(seed: int = 1237) -> Spec:
    """Prefill, 1 sequence L=32768, query chunk = last 8192 tokens; 1% heavy hitters x4."""
    return Spec(name="prefill_L32768_q8192", seq_lens=[32768], nq=[8192], topk=2048,
                heavy_frac=0.01, seed=seed)


def decode_b64_128k(seed: int = 1238) -> Spec:
    """Decode, 64 sequences with L ~ U[64K, 128K]; paged FP8 indexer and FP8 latent KV with
    per-token scales; block/slot tables are seeded random permutations."""
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(65536, 131072 + 1, (64,), generator=g).tolist()
    return Spec(name="decode_b64_ctx64k-128k_fp8kv", seq_lens=lens, nq=[1] * 64, topk=2048,
                kv_fp8=True, permute_tables=True, seed=seed)


def chunked_prefill_128k(chunk: int, seed: int = 1239, n_chunks: int = 16,
                         chunk_q: int = 8192) -> Spec:
    """Chunk ``chunk`` (0-based) of a 131072-token prefill in 16 chunks of 8192 queries:
    the queries are positions [8192*chunk, 8192*(chunk+1)) against the causal prefix.
    FP8 indexer, FP8 latent KV (per-token scale), bf16 q."""
    L = chunk_q * (chunk + 1)
    return Spec(name=f"chunked_prefill_L131072_chunk{chunk}", seq_lens=[L], nq=[chunk_q],
                topk=2048, kv_fp8=True, seed=seed)


CONFIGS = {
    1: tiny_prefill,
    2: decode_b32_8k,
    3: prefill_32k,
    4: decode_b64_128k,
    5: chunked_prefill_128k,
}


# ----------------------------------------------------------------------------------------
# Cache writes: new tokens' indexer keys and latent-KV rows, and where they go.

@dataclass
class StoreSpec:
    """New tokens to write into the two caches: ``n_tokens`` positions 0..n-1 of one
    sequence, their page-64 key rows and page-1 KV slots drawn through seeded
    permutations (a fragmented cache, as after many requests come and go)."""
    name: str
    n_tokens: int
    idx_dim: int = 128
    d_qk: int = 576
    kv_fp8: bool = True            # else a bf16 KV cache
    x_dtype: str = "bf16"          # the new rows' dtype: "bf16" | "f32"
    spare_pages: int = 2           # cache pages / slots that receive nothing
    skip_every: int = 0            # every skip_every-th token has slot -1 (padding)
    heavy_frac: float = 0.01
    heavy_mult: float = 4.0
    seed: int = 1240


@dataclass
class StoreWorkload:
    spec: StoreSpec
    k_new: torch.Tensor            # [n, idx_dim]
    kv_new: torch.Tensor           # [n, d_qk]
    k_slots: torch.Tensor          # [n] int64: physical page * 64 + row, or -1
    kv_slots: torch.Tensor         # [n] int64 slot, or -1
    k_pages: torch.Tensor          # [pages, 64, idx_dim] fp8, pre-filled with a marker code
    k_scale: torch.Tensor          # [pages, 64] fp32, pre-filled with -1
    kv: torch.Tensor               # [slots, d_qk] fp8 or bf16, pre-filled with a marker
    kv_scale: Optional[torch.Tensor]


def make_store(spec: StoreSpec, device="cpu") -> StoreWorkload:
    device = torch.device(device)
    g_cpu = torch.Generator().manual_seed(spec.seed)
    g = torch.Generator(device=device).manual_seed(spec.seed + 1)
    n = spec.n_tokens
    xdt = torch.bfloat16 if spec.x_dtype == "bf16" else torch.float32
    k_new = torch.randn(n, spec.idx_dim, generator=g, device=device)
    kv_new = torch.randn(n, spec.d_qk, generator=g, device=device)
    n_h = int(round(spec.heavy_frac * n))
    if n_h:
        h = torch.randperm(n, generator=g_cpu)[:n_h].to(device)
        k_new[h] *= spec.heavy_mult
        kv_new[h] *= spec.heavy_mult
    pages = (n + INDEXER_PAGE - 1) // INDEXER_PAGE + spec.spare_pages
    page_of = torch.randperm(pages, generator=g_cpu)
    pos = torch.arange(n)
    k_slots = page_of[pos // INDEXER_PAGE].long() * INDEXER_PAGE + pos % INDEXER_PAGE
    n_slots = n + spec.spare_pages * INDEXER_PAGE
    kv_slots = torch.randperm(n_slots, generator=g_cpu)[:n].long()
    if spec.skip_every:
        k_slots[::spec.skip_every] = -1
        kv_slots[::spec.skip_every] = -1
    k_pages = torch.full((pages, INDEXER_PAGE, spec.idx_dim), 0x5A, dtype=torch.uint8,
                         device=device).view(FP8)
    k_scale = torch.full((pages, INDEXER_PAGE), -1.0, device=device)
    if spec.kv_fp8:
        kv = torch.full((n_slots, spec.d_qk), 0x5A, dtype=torch.uint8, device=device).view(FP8)
        kv_scale = torch.full((n_slots,), -1.0, device=device)
    else:
        kv = torch.full((n_slots, spec.d_qk), -3.0, dtype=torch.bfloat16, device=device)
        kv_scale = None
    return StoreWorkload(spec=spec, k_new=k_new.to(xdt), kv_new=kv_new.to(xdt),
                         k_slots=k_slots.to(device), kv_slots=kv_slots.to(device),
                         k_pages=k_pages, k_scale=k_scale, kv=kv, kv_scale=kv_scale)


def store_prompt_128k(seed: int = 1240) -> StoreSpec:
    """A 131072-token prompt's keys and latent KV written into FP8 caches at once
    (bf16 rows in; page-64 key cache and page-1 KV cache, fragmented)."""
    return StoreSpec(name="store_L131072_fp8", n_tokens=131072, seed=seed)


# ----------------------------------------------------------------------------------------
# The whole chunked prefill: one sequence of n_chunks x chunk_q tokens, processed chunk by
# chunk against the growing causal prefix.  Each chunk brings its tokens' new indexer-key
# and latent-KV rows (written into the FP8 caches before the chunk is scored) and its
# queries.

@dataclass
class ChunkedSpec:
    """A prompt of ``n_chunks * chunk_q`` tokens prefilled in chunks of ``chunk_q``."""
    name: str = "chunked_prefill_L131072_16x8192"
    n_chunks: int = 16
    chunk_q: int = 8192
    topk: int = 2048
    idx_heads: int = 64
    idx_dim: int = 128
    w_std: float = 1.0 / 8.0
    heads: int = 128
    d_qk: int = 576
    d_v: int = 512
    softmax_scale: float = 1.0 / math.sqrt(192.0)
    seed: int = 1239

    @property
    def seq_len(self) -> int:
        return self.n_chunks * self.chunk_q

    def chunk_spec(self, c: int) -> Spec:
        """The shape of chunk c as a one-sequence Spec (queries = its chunk_q tokens)."""
        return Spec(name=f"{self.name}_chunk{c}", seq_lens=[self.chunk_q * (c + 1)],
                    nq=[self.chunk_q], topk=self.topk, idx_heads=self.idx_heads,
                    idx_dim=self.idx_dim, w_std=self.w_std, heads=self.heads, d_qk=self.d_qk,
                    d_v=self.d_v, kv_fp8=True, softmax_scale=self.softmax_scale,
                    seed=self.seed)


@dataclass
class ChunkedWorkload:
    spec: ChunkedSpec
    k_new: torch.Tensor            # [L, d_I] bf16: every token's indexer key row
    kv_new: torch.Tensor           # [L, 576] bf16: every token's latent-KV row
    k_slots: torch.Tensor          # [L] int64: page * 64 + row (identity table)
    kv_slots: torch.Tensor         # [L] int64 slot (identity table)
    k_pages: torch.Tensor          # [L/64, 64, d_I] fp8, filled chunk by chunk
    k_scale: torch.Tensor          # [L/64, 64] fp32
    k_block_table: torch.Tensor    # [1, L/64] int32
    kv: torch.Tensor               # [L, 576] fp8, filled chunk by chunk
    kv_scale: torch.Tensor         # [L] fp32
    kv_slot_table: torch.Tensor    # [1, L] int32
    q_idx: torch.Tensor            # [n_chunks, chunk_q, H_I, d_I] fp8
    w: torch.Tensor                # [n_chunks, chunk_q, H_I] fp32
    q: torch.Tensor                # [n_chunks, chunk_q, heads, 576] bf16
    cu_q: torch.Tensor             # [2] int32: (0, chunk_q)
    seq_lens: torch.Tensor         # [n_chunks] int32: chunk_q * (c + 1)

    @property
    def device(self):
        return self.q.device


def make_chunked(spec: ChunkedSpec, device="cpu") -> ChunkedWorkload:
    """Draw the chunked prefill (seeded N(0,1) rows and queries; caches start empty, with a
    marker byte, and identity page / slot tables)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(spec.seed + 1)
    Lt, C, Q = spec.seq_len, spec.n_chunks, spec.chunk_q
    if Lt % INDEXER_PAGE:
        raise ValueError("the prompt length must be a multiple of the indexer page (64)")
    n_pages = Lt // INDEXER_PAGE
    k_new = torch.randn(Lt, spec.idx_dim, generator=g, device=device).to(torch.bfloat16)
    kv_new = torch.randn(Lt, spec.d_qk, generator=g, device=device).to(torch.bfloat16)
    pos = torch.arange(Lt, device=device, dtype=torch.int64)
    q_idx = torch.empty(C, Q, spec.idx_heads, spec.idx_dim, dtype=FP8, device=device)
    w = torch.empty(C, Q, spec.idx_heads, device=device)
    q = torch.empty(C, Q, spec.heads, spec.d_qk, dtype=torch.bfloat16, device=device)
    for c in range(C):          # one chunk at a time bounds the fp32 temporaries
        q_idx[c] = torch.randn(Q, spec.idx_heads, spec.idx_dim, generator=g,
                               device=device).clamp(-FP8_MAX, FP8_MAX).to(FP8)
        w[c] = torch.randn(Q, spec.idx_heads, generator=g, device=device) * spec.w_std
        q[c] = torch.randn(Q, spec.heads, spec.d_qk, generator=g, device=device).to(torch.bfloat16)
    marker = 0x5A
    return ChunkedWorkload(
        spec=spec, k_new=k_new, kv_new=kv_new, k_slots=pos.clone(), kv_slots=pos.clone(),
        k_pages=torch.full((n_pages, INDEXER_PAGE, spec.idx_dim), marker, dtype=torch.uint8,
                           device=device).view(FP8),
        k_scale=torch.full((n_pages, INDEXER_PAGE), -1.0, device=device),
        k_block_table=torch.arange(n_pages, dtype=torch.int32, device=device).reshape(1, -1),
        kv=torch.full((Lt, spec.d_qk), marker, dtype=torch.uint8, device=device).view(FP8),
        kv_scale=torch.full((Lt,), -1.0, device=device),
        kv_slot_table=torch.arange(Lt, dtype=torch.int32, device=device).reshape(1, -1),
        q_idx=q_idx, w=w, q=q,
        cu_q=torch.tensor([0, Q], dtype=torch.int32, device=device),
        seq_lens=torch.tensor([Q * (c + 1) for c in range(C)], dtype=torch.int32, device=device))


def chunk_view(cw: ChunkedWorkload, c: int, k_pages=None, k_scale=None, kv=None,
               kv_scale=None) -> Workload:
    """Chunk c of a chunked prefill as a one-sequence Workload over the whole caches (the
    cache tensors may be replaced, e.g. by copies written elsewhere)."""
    s = cw.spec.chunk_spec(c)
    return Workload(spec=s, cu_q=cw.cu_q, seq_lens=cw.seq_lens[c:c + 1].contiguous(),
                    q_idx=cw.q_idx[c], w=cw.w[c],
                    k_pages=cw.k_pages if k_pages is None else k_pages,
                    k_scale=cw.k_scale if k_scale is None else k_scale,
                    k_block_table=cw.k_block_table, q=cw.q[c],
                    kv=cw.kv if kv is None else kv,
                    kv_scale=cw.kv_scale if kv_scale is None else kv_scale,
                    kv_slot_table=cw.kv_slot_table)
