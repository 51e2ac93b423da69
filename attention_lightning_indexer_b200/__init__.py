"""DeepSeek Sparse Attention (DSA) forward hot path for one B200 (sm_100a).

lightning indexer -> causal top-k -> sparse MLA in MQA mode, as hand-written CUDA
kernels behind the C ABI in ``include/dsa.h`` (``libdsa.so``).  This package is the
thin Python binding: it marshals torch tensors (device memory, streams) into the C
calls and nothing else.
"""
from ._native import (  # noqa: F401
    DSA_BF16,
    DSA_E4M3,
    DSA_E4M3_UE8M0,
    EXPORTED,
    DsaError,
    DsaProblem,
    dsa_cache_write,
    dsa_check_device_errors,
    dsa_dense_mla_fwd,
    dsa_forward,
    dsa_forward_noalloc,
    dsa_forward_noalloc_scratch_bytes,
    dsa_forward_workspace_size,
    dsa_indexer_scores,
    dsa_indexer_topk_streaming,
    dsa_indexer_topk_streaming_workspace_size,
    dsa_sparse_mla_fwd,
    dsa_selftest_bounded_wait,
    dsa_set_debug_checks,
    dsa_topk,
    library_path,
    load,
    make_problem,
    problem_from_inputs,
    scores_ld,
)

__all__ = [
    "DSA_BF16", "DSA_E4M3", "DSA_E4M3_UE8M0", "DsaError", "DsaProblem", "dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_fwd",
    "dsa_indexer_topk_streaming", "dsa_indexer_topk_streaming_workspace_size",
    "dsa_dense_mla_fwd", "dsa_cache_write",
    "dsa_forward_workspace_size", "dsa_forward", "dsa_forward_noalloc", "dsa_forward_noalloc_scratch_bytes",
    "dsa_check_device_errors", "dsa_selftest_bounded_wait", "dsa_set_debug_checks", "make_problem",
    "problem_from_inputs", "scores_ld", "load", "library_path",
]
