"""Host checks of the benchmark's bookkeeping: the algorithmic bytes and flops behind
every reported roofline fraction, against closed forms worked out by hand for the
workload shapes (no GPU needed)."""
import types

import bench
from long_context_sparse_fp8_b200 import workloads as W


def _work(spec, mode):
    return bench.Step.work(types.SimpleNamespace(s=spec, wl=None, mode=mode))


def test_decode_32x8192_counts():
    w = _work(W.decode_b32_8k(), "decode")
    T, L, k = 32, 8192, 2048
    # every selected latent-KV row (bf16 576 + index and slot entry), q, o and lse
    mla_bytes = T * k * (576 * 2 + 8) + T * 128 * 576 * 2 + T * 128 * 512 * 2 + T * 128 * 4
    assert w["mla"]["bytes"] == mla_bytes == 84_951_040
    assert w["mla"]["flops"] == 2 * T * k * 128 * (576 + 512)            # 18.25 GFLOP
    # each key once: 128 B e4m3 + 4 B scale; q_I + w; one fp32 logit per causal pair
    assert w["indexer"]["bytes"] == T * L * 132 + T * 64 * (128 + 4) + T * L * 4
    assert w["indexer"]["flops"] == 2 * T * L * 64 * 128                 # 4.29 GFLOP
    assert w["topk"]["bytes"] == T * L * 4 + T * k * 4


def test_prefill_32k_counts():
    w = _work(W.prefill_32k(), "prefill")
    pairs = sum(range(24577, 32769))                   # query at pos p sees p + 1 keys
    assert pairs == 234_885_120
    assert w["indexer"]["flops"] == 2 * pairs * 64 * 128                 # 3.85 TFLOP
    assert w["mla"]["flops"] == 2 * 8192 * 2048 * 128 * 1088            # 4.67 TFLOP


def test_fp8_kv_row_bytes_and_short_rows():
    spec = W.Spec(name="t", seq_lens=[100, 5000], nq=[2, 1], topk=2048, kv_fp8=True)
    w = _work(spec, "decode")
    n_sel = 99 + 100 + 2048                            # rows shorter than k keep all positions
    q_o = 3 * 128 * (576 + 512) * 2 + 3 * 128 * 4
    assert w["mla"]["bytes"] == n_sel * (576 + 4 + 8) + q_o


def test_sparse_attention_ratio_and_store_bytes():
    assert bench.sparse_ratio(W.decode_b32_8k()) == 0.25
    spec = W.Spec(name="t", seq_lens=[1000], nq=[3], topk=2048)
    assert bench.sparse_ratio(spec) == 1.0            # dense fallback: every key attended
    x = types.SimpleNamespace(shape=(131072, 576), element_size=lambda: 2)
    assert bench._store_bytes(x, 1) == 131072 * (1152 + 576 + 4 + 8) == 228_065_280


def test_chunked_select_blocks_follow_the_workspace():
    """The chunked prefill's launch count restates the library's row-block rule: the
    minimum (L2-sized) workspace gives 148 x 2^m rows per block, a workspace for a whole
    chunk's logits gives one block per chunk (two stores, one indexer, one top-k and one
    attention launch per chunk)."""
    from long_context_sparse_fp8_b200 import chunked as CH
    Q, L = 8192, 131072
    assert CH._block_rows(Q, L) == 148                       # 80 MB / (131072 x 4 B) = 160
    assert CH._block_rows(Q, 8192) == 148 * 16                # 2560 rows fit: 2368
    assert CH._block_rows(Q, 32768) == 592
    assert CH._block_rows(Q, L, Q * L * 4) == Q               # the whole chunk
    assert CH._block_rows(Q, L, 2 * 148 * L * 4 + 100) == 296
    assert CH._block_rows(100, L, 1) == 100                   # fewer rows than a block
    cp = types.SimpleNamespace(batches=[types.SimpleNamespace(total_q=Q, max_seq_len=Q * (c + 1))
                                        for c in range(16)],
                               ws=types.SimpleNamespace(numel=lambda: Q * L * 4))
    assert CH.ChunkedPrefill.launches_per_step(cp) == 16 * 5
    cp.ws = types.SimpleNamespace(numel=lambda: 16)
    assert CH.ChunkedPrefill.launches_per_step(cp) == 1246
