"""libdsa: the DeepSeek Sparse Attention hot path (Lightning Indexer -> top-k ->
sparse MLA) as hand-written sm_100a CUDA kernels behind a C ABI (include/dsa.h).

``long_context_sparse_fp8_b200.dsa`` is the ctypes binding; ``workloads`` draws
seeded synthetic inputs.
"""
from . import dsa  # noqa: F401
from .dsa import (Batch, DsaError, PagedCache, dsa_cache_store, dsa_decode, dsa_decode_workspace_size,  # noqa: F401
                  dsa_device_check, dsa_indexer_logits, dsa_indexer_topk,
                  dsa_indexer_topk_workspace_size, dsa_sparse_mla_decode,
                  dsa_sparse_mla_decode_noalloc,
                  dsa_sparse_mla_decode_workspace_size, dsa_sparse_mla_prefill, dsa_topk,
                  dsa_version, load_library)
