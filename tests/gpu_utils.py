"""Shared helpers for the GPU parity tests: seeded inputs on the device, row sampling,
and the comparison rules (tolerances written out here, used by every parity test).

Tolerances (from the stated parity bar):
  * top-k indices: bit-exact given the same fp32 score array (ties -> smaller index);
  * indexer scores: |gpu - oracle| <= 1e-3 * sum_j |w[t,j]| * sum_d |q[t,j,d] * k[s,d]|;
  * selected sets end to end: recall >= 0.999 after removing keys whose oracle score is
    within that tolerance of the k-th oracle score (near ties);
  * attention output: max |o_gpu - o_oracle| <= 2e-2 for the same index set;
    lse: |lse_gpu - lse_oracle| <= 2e-3 (fp32 softmax statistics over <= 2048 logits
    computed from bf16 products with fp32 accumulation).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

SCORE_RTOL = 1e-3
O_ATOL = 2e-2
LSE_ATOL = 2e-3
RECALL_MIN = 0.999


def sample_rows(T: int, k: int, n_rand: int, seed: int = 0, edge: int = 16) -> np.ndarray:
    """First `edge` rows, a band around t = k, the last `edge` rows and seeded random rows."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(edge, T)))
    rows |= set(range(max(0, k - edge // 2), min(T, k + edge // 2)))
    rows |= set(range(max(0, T - edge), T))
    rows |= set(rng.integers(0, T, n_rand).tolist()) if T > 0 else set()
    return np.array(sorted(rows), dtype=np.int64)


def score_bound_row(q_row: torch.Tensor, w_row: torch.Tensor, k_rows: torch.Tensor) -> np.ndarray:
    """sum_j |w[j]| * sum_d |q[j,d] k[s,d]| for one query row against k_rows [n, D] (fp64).

    q_row / k_rows are the (dequantised) values; the bound is the tolerance scale."""
    a = q_row.double().abs() @ k_rows.double().abs().T       # [H, n]
    return (w_row.double().abs() @ a).numpy()


def fp8_to_f64(codes: torch.Tensor) -> torch.Tensor:
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


def assert_scores_close(gpu_rows: np.ndarray, ora_rows: np.ndarray, bound, pos: np.ndarray):
    """bound[r] holds the tolerance scale of keys 0..pos[r] of row r."""
    for r in range(gpu_rows.shape[0]):
        n = int(pos[r]) + 1
        err = np.abs(gpu_rows[r, :n].astype(np.float64) - ora_rows[r, :n])
        lim = SCORE_RTOL * np.asarray(bound[r])[:n] + 1e-30
        bad = np.nonzero(err > lim)[0]
        assert bad.size == 0, f"row {r}: {bad.size} scores off, worst err {err.max():.3e} vs lim {lim[bad[0]]:.3e}"


def recall_excluding_near_ties(gpu_idx: np.ndarray, ora_scores: np.ndarray, bound, pos: np.ndarray, k: int):
    """Recall of the 'certainly selected' keys and count of 'certainly excluded' keys picked."""
    hits = total = wrong = 0
    for r in range(gpu_idx.shape[0]):
        n = int(pos[r]) + 1
        sc = ora_scores[r, :n]
        keff = min(k, n)
        sel = set(int(x) for x in gpu_idx[r] if x >= 0)
        assert len(sel) == keff, f"row {r}: {len(sel)} distinct indices, expected {keff}"
        npad = int(np.count_nonzero(gpu_idx[r] == -1))
        assert npad == k - keff, f"row {r}: {npad} slots of -1 padding, expected {k - keff}"
        assert max(sel) <= n - 1
        if keff == n:
            assert sel == set(range(n))
            continue
        kth = np.sort(sc)[::-1][keff - 1]
        tol = SCORE_RTOL * np.asarray(bound[r])[:n]
        certain_in = np.nonzero(sc > kth + tol)[0]
        certain_out = np.nonzero(sc < kth - tol)[0]
        hits += sum(1 for s in certain_in if int(s) in sel)
        total += len(certain_in)
        wrong += sum(1 for s in certain_out if int(s) in sel)
    return (hits / total if total else 1.0), wrong


def sorted_rows(idx: np.ndarray) -> np.ndarray:
    """Each row sorted ascending with -1 padding moved to the end (order is unspecified)."""
    out = np.sort(np.where(idx < 0, np.iinfo(np.int32).max, idx), axis=1)
    return np.where(out == np.iinfo(np.int32).max, -1, out)
