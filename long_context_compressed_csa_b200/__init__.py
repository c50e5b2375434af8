"""B200-native CSA / HCA hot path (DeepSeek-V4 hybrid attention), Python binding.

Thin ctypes marshalling over ``libcsa_b200.so`` (C ABI declared in ``include/csa.h``):
every function takes torch CUDA tensors, passes their device pointers, sizes and the
current CUDA stream to the library entry point of the same name, and raises on a
non-zero status.  No computation happens here and there is no fallback: if the library
is missing, importing the functions raises.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    CSAError,
    csa_attn_workspace_size,
    csa_compress,
    csa_indexer_topk,
    csa_indexer_topk_e2m1,
    csa_indexer_topk_e4m3,
    csa_indexer_topk_noalloc,
    csa_indexer_topk_noalloc_status,
    csa_indexer_topk_workspace_size,
    csa_quantize_e2m1,
    csa_quantize_e4m3,
    csa_sparse_attn,
    csa_status_string,
    csa_version,
    csa_workspace_set_wait_budget,
    csa_workspace_status,
    csa_workspace_zero,
    hca_compress,
    hca_project_compress,
    csa_project_compress,
    hca_dense_attn,
    library,
    library_path,
)
