"""ctypes binding of libdsa.so (C ABI in include/dsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
The functions keep the C names and take torch tensors (device memory owned by the
caller) plus the current CUDA stream.  If the library is missing or cannot load, the
call raises -- there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

DSA_BF16 = 0
DSA_E4M3 = 1
DSA_E4M3_UE8M0 = 2

_STATUS = {
    0: "DSA_OK",
    1: "DSA_ERR_INVALID_ARG",
    2: "DSA_ERR_UNSUPPORTED",
    3: "DSA_ERR_WORKSPACE",
    4: "DSA_ERR_CUDA",
    5: "DSA_ERR_DEVICE_TIMEOUT",
    6: "DSA_ERR_DEVICE_BOUNDS",
}

EXPORTED = (
    "dsa_indexer_scores",
    "dsa_topk",
    "dsa_indexer_topk_streaming_workspace_size",
    "dsa_indexer_topk_streaming",
    "dsa_sparse_mla_fwd",
    "dsa_dense_mla_fwd",
    "dsa_forward_workspace_size",
    "dsa_forward",
    "dsa_forward_noalloc",
    "dsa_forward_noalloc_scratch_bytes",
    "dsa_check_device_errors",
    "dsa_cache_write",
    "dsa_set_debug_checks",
    "dsa_selftest_bounded_wait",
    "dsa_status_string",
    "dsa_abi_version",
)


class DsaError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {_STATUS.get(code, code)} ({msg})")
        self.code = code


class DsaProblem(ctypes.Structure):
    """Mirror of ``dsa_problem_t``."""

    _fields_ = [
        ("batch", ctypes.c_int32),
        ("cu_q", ctypes.c_void_p),
        ("cu_k", ctypes.c_void_p),
        ("total_q", ctypes.c_int32),
        ("total_k", ctypes.c_int32),
        ("max_len_q", ctypes.c_int32),
        ("max_len_k", ctypes.c_int32),
        ("n_idx_heads", ctypes.c_int32),
        ("idx_dim", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("d_qk", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("idx_dtype", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
        ("block_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
    ]


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libdsa.so (building it first when it is missing or stale and nvcc exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing and _build.needs_build():
        _build.build()
    if not os.path.exists(_build.LIB):
        raise RuntimeError(f"libdsa.so not found at {_build.LIB}; run python -m attention_lightning_indexer_b200.build")
    lib = ctypes.CDLL(_build.LIB)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    pp = ctypes.POINTER(DsaProblem)
    lib.dsa_indexer_scores.argtypes = [pp, P, P, P, P, P, P, i64, i32, i32, P]
    lib.dsa_topk.argtypes = [pp, P, i64, i32, i32, P, P]
    lib.dsa_indexer_topk_streaming_workspace_size.argtypes = [pp, i32]
    lib.dsa_indexer_topk_streaming_workspace_size.restype = sz
    lib.dsa_indexer_topk_streaming.argtypes = [pp, P, P, P, P, P, i32, i32, i32, P, P, sz, P]
    lib.dsa_sparse_mla_fwd.argtypes = [pp, P, P, P, P, P, P]
    lib.dsa_dense_mla_fwd.argtypes = [pp, P, P, P, P, P, P]
    lib.dsa_forward_workspace_size.argtypes = [pp, i32]
    lib.dsa_forward_workspace_size.restype = sz
    lib.dsa_forward.argtypes = [pp, P, P, P, P, P, P, P, i32, P, P, P, P, sz, P]
    lib.dsa_forward_noalloc.argtypes = [pp, P, P, P, P, P, P, P, P, P, P, P]
    lib.dsa_forward_noalloc_scratch_bytes.argtypes = []
    lib.dsa_forward_noalloc_scratch_bytes.restype = sz
    lib.dsa_check_device_errors.argtypes = [P]
    lib.dsa_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P]
    lib.dsa_cache_write.argtypes = [i32, P, P, P, P, P, P, P, P, ctypes.c_float, P, P, P]
    lib.dsa_set_debug_checks.argtypes = [i32]
    lib.dsa_set_debug_checks.restype = None
    lib.dsa_status_string.argtypes = [ctypes.c_int]
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_abi_version.restype = i32
    for name in ("dsa_indexer_scores", "dsa_topk", "dsa_indexer_topk_streaming", "dsa_sparse_mla_fwd", "dsa_dense_mla_fwd", "dsa_forward",
                 "dsa_forward_noalloc",
                 "dsa_check_device_errors", "dsa_selftest_bounded_wait", "dsa_cache_write"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(code: int, where: str) -> None:
    if code != 0:
        raise DsaError(code, where, load().dsa_status_string(code).decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libdsa takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_problem(batch: int, total_q: int, total_k: int, max_len_q: int, max_len_k: int, topk: int,
                 cu_q: Optional[torch.Tensor] = None, cu_k: Optional[torch.Tensor] = None,
                 idx_dtype: int = DSA_BF16, sm_scale: float = 1.0 / 192 ** 0.5,
                 n_idx_heads: int = 64, idx_dim: int = 128, n_heads: int = 128, d_qk: int = 576,
                 d_v: int = 512, block_table: Optional[torch.Tensor] = None, page_size: int = 64) -> DsaProblem:
    if cu_q is not None:
        assert cu_q.dtype == torch.int32 and cu_k is not None and cu_k.dtype == torch.int32
    max_pages = 0
    if block_table is not None:
        assert block_table.dtype == torch.int32 and block_table.dim() == 2
        max_pages = block_table.shape[1]
    return DsaProblem(batch, _ptr(cu_q), _ptr(cu_k), total_q, total_k, max_len_q, max_len_k, n_idx_heads,
                      idx_dim, n_heads, d_qk, d_v, topk, idx_dtype, sm_scale, _ptr(block_table), page_size,
                      max_pages)


def problem_from_inputs(inp: dict, sm_scale: float = 1.0 / 192 ** 0.5) -> DsaProblem:
    """dsa_problem_t for a dict produced by the seeded input generators (tensors on the GPU)."""
    fp8 = "q_idx8" in inp
    blocks = "q_scale_ue8m0" in inp
    paged = "block_table" in inp
    cu_q = inp.get("cu_q") if inp["batch"] > 1 or paged else None
    cu_k = inp.get("cu_k") if inp["batch"] > 1 or paged else None
    total_k = inp["phys_k"] if paged else inp["total_k"]
    return make_problem(inp["batch"], inp["total_q"], total_k, inp["max_len_q"], inp["max_len_k"],
                        inp["topk"], cu_q=cu_q, cu_k=cu_k,
                        idx_dtype=(DSA_E4M3_UE8M0 if blocks else DSA_E4M3) if fp8 else DSA_BF16,
                        sm_scale=sm_scale, block_table=inp.get("block_table"), page_size=inp.get("page_size", 64))


def scores_ld(max_len_k: int) -> int:
    return max(4, (max_len_k + 3) // 4 * 4)


# ---------------------------------------------------------------- entry points

def dsa_indexer_scores(p: DsaProblem, q_idx, k_idx, w, scores, row_begin: int = 0, row_count: Optional[int] = None,
                       q_scale=None, k_scale=None, stream=None) -> None:
    lib = load()
    if row_count is None:
        row_count = p.total_q - row_begin
    _check(lib.dsa_indexer_scores(ctypes.byref(p), _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w),
                                  _ptr(scores), scores.stride(0), row_begin, row_count, _stream(stream)),
           "dsa_indexer_scores")


def dsa_topk(p: DsaProblem, scores, idx, row_begin: int = 0, row_count: Optional[int] = None, stream=None) -> None:
    lib = load()
    if row_count is None:
        row_count = p.total_q - row_begin
    _check(lib.dsa_topk(ctypes.byref(p), _ptr(scores), scores.stride(0), row_begin, row_count, _ptr(idx),
                        _stream(stream)), "dsa_topk")


def dsa_indexer_topk_streaming_workspace_size(p: DsaProblem, chunk_q: int = 0) -> int:
    return int(load().dsa_indexer_topk_streaming_workspace_size(ctypes.byref(p), chunk_q))


def dsa_indexer_topk_streaming(p: DsaProblem, q_idx, k_idx, w, idx, workspace, row_begin: int = 0,
                               row_count: Optional[int] = None, chunk_q: int = 0, q_scale=None, k_scale=None,
                               stream=None) -> None:
    """Indexer and top-k without score rows: the same idx as dsa_indexer_scores + dsa_topk."""
    lib = load()
    if row_count is None:
        row_count = p.total_q - row_begin
    _check(lib.dsa_indexer_topk_streaming(ctypes.byref(p), _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale),
                                          _ptr(w), row_begin, row_count, chunk_q, _ptr(idx), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)),
           "dsa_indexer_topk_streaming")


def dsa_sparse_mla_fwd(p: DsaProblem, q, kv, idx, out, lse, stream=None) -> None:
    lib = load()
    _check(lib.dsa_sparse_mla_fwd(ctypes.byref(p), _ptr(q), _ptr(kv), _ptr(idx), _ptr(out), _ptr(lse),
                                  _stream(stream)), "dsa_sparse_mla_fwd")


def dsa_dense_mla_fwd(p: DsaProblem, q, kv, idx, out, lse, stream=None) -> None:
    """Dense (masked MHA) form: all causal keys, restricted to idx's keys when idx is given."""
    lib = load()
    _check(lib.dsa_dense_mla_fwd(ctypes.byref(p), _ptr(q), _ptr(kv), _ptr(idx), _ptr(out), _ptr(lse),
                                 _stream(stream)), "dsa_dense_mla_fwd")


def dsa_forward_workspace_size(p: DsaProblem, chunk_q: int = 0) -> int:
    return int(load().dsa_forward_workspace_size(ctypes.byref(p), chunk_q))


def dsa_forward(p: DsaProblem, q_idx, k_idx, w, q, kv, out, lse, workspace, chunk_q: int = 0, idx_out=None,
                q_scale=None, k_scale=None, stream=None) -> None:
    lib = load()
    _check(lib.dsa_forward(ctypes.byref(p), _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w), _ptr(q),
                           _ptr(kv), chunk_q, _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream)), "dsa_forward")


def dsa_forward_noalloc(p: DsaProblem, q_idx, k_idx, w, q, kv, idx_out, out, lse, q_scale=None, k_scale=None,
                        stream=None) -> None:
    """dsa_forward with the library's fixed scratch array instead of a caller workspace (no
    device allocation by the call; see include/dsa.h for the size limit and sharing rules)."""
    lib = load()
    _check(lib.dsa_forward_noalloc(ctypes.byref(p), _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w),
                                   _ptr(q), _ptr(kv), _ptr(idx_out), _ptr(out), _ptr(lse), _stream(stream)),
           "dsa_forward_noalloc")


def dsa_forward_noalloc_scratch_bytes() -> int:
    return int(load().dsa_forward_noalloc_scratch_bytes())


def dsa_check_device_errors(stream=None) -> None:
    _check(load().dsa_check_device_errors(_stream(stream)), "dsa_check_device_errors")


def dsa_cache_write(k_idx_raw, kv_raw, positions, rows, k_norm_w, k_norm_b, kv_norm_w, inv_freq, k_idx_cache,
                    kv_cache, eps: float = 1e-6, stream=None) -> None:
    """Indexer-key and latent cache rows of new tokens (norms + RoPE; see include/dsa.h)."""
    lib = load()
    _check(lib.dsa_cache_write(int(positions.numel()), _ptr(k_idx_raw), _ptr(kv_raw), _ptr(positions), _ptr(rows),
                               _ptr(k_norm_w), _ptr(k_norm_b), _ptr(kv_norm_w), _ptr(inv_freq), eps,
                               _ptr(k_idx_cache), _ptr(kv_cache), _stream(stream)), "dsa_cache_write")


def dsa_set_debug_checks(enable: bool) -> None:
    """Per-row input checks in every kernel (see include/dsa.h)."""
    load().dsa_set_debug_checks(1 if enable else 0)


def dsa_selftest_bounded_wait(limit_us: int = 1000, stream=None) -> None:
    """Launch the one-CTA kernel whose bounded wait runs out (see include/dsa.h)."""
    _check(load().dsa_selftest_bounded_wait(limit_us, _stream(stream)), "dsa_selftest_bounded_wait")
