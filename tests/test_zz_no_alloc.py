"""dsa_sparse_mla_decode_noalloc (split partials in the library's fixed device array)
against dsa_sparse_mla_decode (caller workspace), through the C ABI.

Collected last on purpose: the array keeps whatever earlier calls left in it, and the
comparison must hold after the other tests have run as well as alone.  Three shapes: the
tensor-core split path (fp16 partials), the CUDA-core split path (fp32 partials) and a
batch large enough that the rows are not split at all (no scratch used).
"""
import math

import pytest
import torch

import long_context_sparse_fp8_b200 as L
from long_context_sparse_fp8_b200 import workloads as W

from _helpers import (MLA_ATOL_BF16, MLA_ATOL_F32, check_mla, lib_args, run_indexer, run_mla,
                      run_topk)


def _noalloc(wl, idx):
    s = wl.spec
    batch, _, kv = lib_args(wl)
    dt = torch.bfloat16 if s.mla_dtype == "bf16" else torch.float32
    out = torch.full((s.total_q, s.heads, s.d_v), float("nan"), dtype=dt, device=wl.device)
    lse = torch.full((s.total_q, s.heads), float("nan"), device=wl.device)
    L.dsa_sparse_mla_decode_noalloc(wl.q, kv, batch, idx, s.d_v, s.softmax_scale, out, lse)
    return out, lse


def _spec(kind):
    if kind == "tc_split":         # 32 rows x 2048: split in two, fp16 partials
        return W.decode_b32_8k(), MLA_ATOL_BF16, True
    if kind == "f32_split":        # CUDA-core attention, 2 rows split eight ways
        return W.Spec(name="f32_split", seq_lens=[3000, 2500], nq=[1, 1], topk=2048, idx_heads=4,
                      idx_dim=32, idx_fp8=False, w_std=0.5, heads=2, d_qk=80, d_v=64,
                      mla_dtype="f32", softmax_scale=1.0 / math.sqrt(80.0), seed=7), MLA_ATOL_F32, True
    return W.Spec(name="no_split", seq_lens=[3000] * 40, nq=[1] * 40, topk=2048, seed=8), \
        MLA_ATOL_BF16, False


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["tc_split", "f32_split", "no_split"])
def test_noalloc_matches_workspace_decode_twice(kind):
    spec, atol, splits = _spec(kind)
    wl = W.make(spec, "cuda")
    s = wl.spec
    assert (L.dsa_sparse_mla_decode_workspace_size(s.total_q, s.heads, s.d_v, s.topk) > 0) == splits
    idx = run_topk(wl, run_indexer(wl))
    ref_out, ref_lse = run_mla(wl, idx, decode=True)
    ref_out = ref_out.float().cpu().numpy()
    ref_lse = ref_lse.cpu().numpy()
    for _ in range(2):
        out, lse = _noalloc(wl, idx)
        torch.cuda.synchronize()
        assert L.dsa_device_check() == 0
        check_mla(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, atol)
