"""fp64 CPU oracle for the DSA forward path (lightning indexer -> top-k -> sparse MLA).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``; never by the product
package.  The arithmetic lives in ``dsa_oracle.c`` (plain C, fp64, OpenMP over query
rows); this module only builds it, marshals numpy arrays and turns bf16/fp32 tensors
into fp64 (an exact widening).  The method's definition and the readings of the pages
are stated in the C file's header.

Pinning status (what ties each function to the pages rather than to itself) is listed
in ``tests/test_oracle_pins.py``; every function below has at least one pin there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")

_lib: Optional[ctypes.CDLL] = None


def build(force: bool = False) -> str:
    """Compile ``dsa_oracle.c`` into ``libdsa_oracle.so`` beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.dsa_oracle_indexer.argtypes = [i32, P, P, P, P, i32, i32, i32, P, P, P, i64]
        lib.dsa_oracle_indexer_fp8.argtypes = [i32, P, P, P, i32, P, P, P, i32, i32, i32, P, P, P, i64]
        lib.dsa_oracle_ue8m0_value.argtypes = [ctypes.c_uint8]
        lib.dsa_oracle_ue8m0_value.restype = f64
        lib.dsa_oracle_topk.argtypes = [i32, P, P, i64, i32, i32, P, P, P]
        lib.dsa_oracle_sparse_mla.argtypes = [i32, P, P, P, i32, P, i32, i32, i32, f64, i32, P, P, P, P]
        lib.dsa_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.dsa_oracle_e4m3_value.restype = f64
        lib.dsa_oracle_num_threads.restype = i32
        lib.dsa_oracle_set_pages.argtypes = [P, i32, i32]
        lib.dsa_oracle_cache_write.argtypes = [i32, P, P, P, P, P, P, P, f64, P, P]
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().dsa_oracle_num_threads())


class _Pages:
    """Key rows through a block table (paged caches) for the duration of one call."""

    def __init__(self, block_table, page_size: int):
        self.table = None if block_table is None else _np(block_table, np.int32)
        self.page = page_size

    def __enter__(self):
        if self.table is not None:
            _load().dsa_oracle_set_pages(_ptr(self.table), self.table.shape[1], self.page)
        return self

    def __exit__(self, *exc):
        _load().dsa_oracle_set_pages(None, 0, 0)
        return False


# ---------------------------------------------------------------- marshalling

def _np(x, dtype) -> np.ndarray:
    """Host numpy array of ``dtype`` (C-contiguous).  Accepts torch tensors on any device."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach()
            if x.dtype in (torch.bfloat16, torch.float16):
                x = x.float()
            if x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8)
            x = x.cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _cu(cu, n_default: int) -> np.ndarray:
    if cu is None:
        return np.array([0, n_default], dtype=np.int32)
    return _np(cu, np.int32)


def _rows(rows, total_q: int) -> np.ndarray:
    if rows is None:
        return np.arange(total_q, dtype=np.int64)
    return _np(rows, np.int64)


# ---------------------------------------------------------------- public calls

def indexer(q_rows, w_rows, k, rows=None, cu_q=None, cu_k=None, ld: Optional[int] = None,
            block_table=None, page_size: int = 64) -> np.ndarray:
    """Index scores I[r, s] for the listed query rows (fp64; -inf where s > pos(t)).

    q_rows [R, H, D], w_rows [R, H] are the listed rows' query vectors and weights;
    k [S_total, D].  Without ``cu_q``/``cu_k`` the problem is one sequence with
    queries = keys (plain prefill).  With ``block_table`` [B, max_pages] the keys are
    paged: key s of sequence b is row table[b, s // page_size] * page_size + s % page_size
    of k (``cu_k`` then only gives the sequence lengths).
    """
    q = _np(q_rows, np.float64)
    w = _np(w_rows, np.float64)
    kk = _np(k, np.float64)
    R, H, D = q.shape
    cuq = _cu(cu_q, kk.shape[0])
    cuk = _cu(cu_k, kk.shape[0])
    rr = _rows(rows, R)
    batch = len(cuk) - 1
    if ld is None:
        ld = int(np.max(np.diff(cuk))) if batch > 0 else 0
    out = np.empty((R, ld), dtype=np.float64)
    with _Pages(block_table, page_size):
        _load().dsa_oracle_indexer(R, _ptr(rr), _ptr(q), _ptr(w), _ptr(kk), H, D, batch,
                                   _ptr(cuq), _ptr(cuk), _ptr(out), ld)
    return out


def indexer_fp8(q8_rows, q_scale_rows, w_rows, k8, k_scale, rows=None, cu_q=None, cu_k=None,
                ld: Optional[int] = None, block_table=None, page_size: int = 64) -> np.ndarray:
    """FP8 variant of :func:`indexer`: e4m3 codes with per-token fp32 scales
    (q_scale_rows [R], k_scale [S]) or per-(token, head) q scales (q_scale_rows [R, H])."""
    q8 = _np(q8_rows, np.uint8)
    qs = _np(q_scale_rows, np.float64)
    per_head = 1 if qs.ndim == 2 else 0
    w = _np(w_rows, np.float64)
    k8a = _np(k8, np.uint8)
    ks = _np(k_scale, np.float64)
    R, H, D = q8.shape
    cuq = _cu(cu_q, k8a.shape[0])
    cuk = _cu(cu_k, k8a.shape[0])
    rr = _rows(rows, R)
    batch = len(cuk) - 1
    if ld is None:
        ld = int(np.max(np.diff(cuk))) if batch > 0 else 0
    out = np.empty((R, ld), dtype=np.float64)
    with _Pages(block_table, page_size):
        _load().dsa_oracle_indexer_fp8(R, _ptr(rr), _ptr(q8), _ptr(qs), per_head, _ptr(w), _ptr(k8a), _ptr(ks),
                                       H, D, batch, _ptr(cuq), _ptr(cuk), _ptr(out), ld)
    return out


def ue8m0_value(code: int) -> float:
    return float(_load().dsa_oracle_ue8m0_value(int(code) & 0xFF))


def ue8m0_decode(codes) -> np.ndarray:
    """Scale bytes (ue8m0, any shape) to fp64 values through the oracle's decoder."""
    c = _np(codes, np.uint8)
    table = np.array([ue8m0_value(i) for i in range(256)], dtype=np.float64)
    return table[c]


def indexer_fp8_block(q8_rows, q_scale_codes_rows, w_rows, k8, k_scale_codes, **kw) -> np.ndarray:
    """FP8 indexer with ue8m0 block scales: q_scale_codes_rows [R, H], k_scale_codes [S] bytes."""
    return indexer_fp8(q8_rows, ue8m0_decode(q_scale_codes_rows), w_rows, k8, ue8m0_decode(k_scale_codes), **kw)


def e4m3_value(code: int) -> float:
    return float(_load().dsa_oracle_e4m3_value(int(code) & 0xFF))


def topk(scores, k: int, rows=None, cu_q=None, cu_k=None) -> np.ndarray:
    """Top-k indices per listed row, best first, -1 padded ([R, k] int32).

    ``scores`` [R, ld] is read as values (fp32 arrays are widened exactly)."""
    s = _np(scores, np.float64)
    R, ld = s.shape
    cuq = _cu(cu_q, ld)
    cuk = _cu(cu_k, ld)
    rr = _rows(rows, R)
    batch = len(cuk) - 1
    out = np.empty((R, k), dtype=np.int32)
    _load().dsa_oracle_topk(R, _ptr(rr), _ptr(s), ld, k, batch, _ptr(cuq), _ptr(cuk), _ptr(out))
    return out


def sparse_mla(q_rows, kv, idx_rows, scale: float, d_v: int = 512, rows=None, cu_q=None, cu_k=None,
               block_table=None, page_size: int = 64):
    """Sparse MLA (MQA mode) for the listed rows: returns (o [R,H,d_v], lse [R,H]) in fp64."""
    q = _np(q_rows, np.float64)
    kva = _np(kv, np.float64)
    ix = _np(idx_rows, np.int32)
    R, H, Dqk = q.shape
    k = ix.shape[1]
    cuq = _cu(cu_q, kva.shape[0])
    cuk = _cu(cu_k, kva.shape[0])
    rr = _rows(rows, R)
    batch = len(cuk) - 1
    o = np.empty((R, H, d_v), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    with _Pages(block_table, page_size):
        _load().dsa_oracle_sparse_mla(R, _ptr(rr), _ptr(q), _ptr(ix), k, _ptr(kva), H, Dqk, d_v,
                                      float(scale), batch, _ptr(cuq), _ptr(cuk), _ptr(o), _ptr(lse))
    return o, lse


def forward(q_idx_rows, w_rows, k_idx, q_rows, kv, topk_k: int, scale: float, d_v: int = 512,
            rows=None, cu_q=None, cu_k=None, block_table=None, page_size: int = 64):
    """The whole path for the listed rows, all in fp64: indexer -> top-k -> sparse MLA.

    Returns (scores, idx, o, lse)."""
    sc = indexer(q_idx_rows, w_rows, k_idx, rows=rows, cu_q=cu_q, cu_k=cu_k, block_table=block_table,
                 page_size=page_size)
    ix = topk(sc, topk_k, rows=rows, cu_q=cu_q, cu_k=cu_k)
    o, lse = sparse_mla(q_rows, kv, ix, scale, d_v=d_v, rows=rows, cu_q=cu_q, cu_k=cu_k, block_table=block_table,
                        page_size=page_size)
    return sc, ix, o, lse


def positions(rows: Sequence[int], cu_q, cu_k) -> np.ndarray:
    """pos(t) of each listed row under the boundary's reading (queries are the last tokens)."""
    cuq = _np(cu_q, np.int64)
    cuk = _np(cu_k, np.int64)
    out = []
    for t in rows:
        b = int(np.searchsorted(cuq, t, side="right") - 1)
        out.append((cuk[b + 1] - cuk[b]) - (cuq[b + 1] - cuq[b]) + (t - cuq[b]))
    return np.array(out, dtype=np.int64)


def cache_write(k_raw, kv_raw, positions, ln_w, ln_b, rms_w, inv_freq, eps: float):
    """Indexer key and latent rows of new tokens (k_norm + non-interleaved RoPE; RMSNorm +
    interleaved RoPE on the latent's RoPE dims): returns (k [n, 128], kv [n, 576]) in fp64."""
    kr = _np(k_raw, np.float64)
    zr = _np(kv_raw, np.float64)
    n = kr.shape[0]
    ps = _np(positions, np.int32)
    out_k = np.empty((n, 128), dtype=np.float64)
    out_kv = np.empty((n, 576), dtype=np.float64)
    _load().dsa_oracle_cache_write(n, _ptr(kr), _ptr(zr), _ptr(ps), _ptr(_np(ln_w, np.float64)),
                                   _ptr(_np(ln_b, np.float64)), _ptr(_np(rms_w, np.float64)),
                                   _ptr(_np(inv_freq, np.float64)), float(eps), _ptr(out_k), _ptr(out_kv))
    return out_k, out_kv
