"""dsa_sparse_mla_decode_noalloc (split partials in the library's fixed device array)
against dsa_sparse_mla_decode (caller workspace), through the C ABI.

Collected last on purpose: the array keeps whatever earlier calls left in it, and the
comparison must hold after the other tests have run as well as alone.
"""
import pytest
import torch

import long_context_sparse_fp8_b200 as L
from long_context_sparse_fp8_b200 import workloads as W

from _helpers import MLA_ATOL_BF16, check_mla, lib_args, run_indexer, run_mla, run_topk


def _noalloc(wl, idx):
    s = wl.spec
    batch, _, kv = lib_args(wl)
    out = torch.full((s.total_q, s.heads, s.d_v), float("nan"), dtype=torch.bfloat16,
                     device=wl.device)
    lse = torch.full((s.total_q, s.heads), float("nan"), device=wl.device)
    L.dsa_sparse_mla_decode_noalloc(wl.q, kv, batch, idx, s.d_v, s.softmax_scale, out, lse)
    return out, lse


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_twice():
    wl = W.make(W.decode_b32_8k(), "cuda")
    s = wl.spec
    assert L.dsa_sparse_mla_decode_workspace_size(s.total_q, s.heads, s.d_v, s.topk) > 0
    idx = run_topk(wl, run_indexer(wl))
    ref_out, ref_lse = run_mla(wl, idx, decode=True)
    ref_out = ref_out.float().cpu().numpy()
    ref_lse = ref_lse.cpu().numpy()
    for _ in range(2):
        out, lse = _noalloc(wl, idx)
        torch.cuda.synchronize()
        assert L.dsa_device_check() == 0
        check_mla(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, MLA_ATOL_BF16)
