"""dsa_forward_noalloc -- the entry point for callers that cannot allocate device memory
where they run the path (host callbacks, runtimes that own all device memory, serving
loops that must not call cudaMalloc) -- against dsa_forward with a caller workspace.

The variant keeps its score scratch in a fixed 32 MiB array inside the library, so it
takes no workspace argument.  This file is named to be collected last: if it fails, a
run that stops at the first failure has already run every other test.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import attention_lightning_indexer_b200 as dsa
import dsa_synth
from gpu_utils import LSE_ATOL, O_ATOL, sorted_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(inp):
    T = inp["total_q"]
    return (torch.empty((T, inp["topk"]), dtype=torch.int32, device=DEV),
            torch.empty((T, 128, 512), dtype=torch.bfloat16, device=DEV),
            torch.empty((T, 128), dtype=torch.float32, device=DEV))


def _with_workspace(inp):
    p = dsa.problem_from_inputs(inp)
    idx, out, lse = _outputs(inp)
    ws = torch.empty(dsa.dsa_forward_workspace_size(p, 0), dtype=torch.uint8, device=DEV)
    dsa.dsa_forward(p, inp["q_idx"], inp["k_idx"], inp["w"], inp["q"], inp["kv"], out, lse, ws, idx_out=idx)
    return idx, out, lse


def _without_allocation(inp):
    p = dsa.problem_from_inputs(inp)
    idx, out, lse = _outputs(inp)
    dsa.dsa_forward_noalloc(p, inp["q_idx"], inp["k_idx"], inp["w"], inp["q"], inp["kv"], idx, out, lse)
    return idx, out, lse


def _assert_same(ref, got):
    (ri, ro, rl), (gi, go, gl) = ref, got
    np.testing.assert_array_equal(sorted_rows(gi.cpu().numpy()), sorted_rows(ri.cpu().numpy()))
    assert torch.max(torch.abs(go.float() - ro.float())).item() <= O_ATOL
    fin = torch.isfinite(rl)
    assert torch.equal(fin, torch.isfinite(gl))
    assert torch.max(torch.abs(gl[fin] - rl[fin])).item() <= LSE_ATOL


def test_noalloc_matches_workspace_forward_on_two_calls_in_a_row():
    # 1st call: one 9000-token prefill -- its 36 KB score rows need ~10 chunks of the
    # fixed scratch.  2nd call right after, on a ragged batch, starts from the scratch
    # contents the first call left behind.
    first = dsa_synth.make_prefill(9000, topk=256, seed=41, device=DEV)
    second = dsa_synth.make_decode(5, 700, 4000, topk=512, seed=42, device=DEV, q_per_seq=3)
    assert 9000 * 4 * 1000 > dsa.dsa_forward_noalloc_scratch_bytes()   # really chunked
    for inp in (first, second):
        ref = _with_workspace(inp)
        got = _without_allocation(inp)
        torch.cuda.synchronize()
        _assert_same(ref, got)
    dsa.dsa_check_device_errors()


def test_noalloc_rejects_rows_longer_than_its_scratch():
    # One score row of 9M keys (36 MB) cannot fit in the 32 MiB array: rejected on the
    # host, before any launch (the pointers below are never dereferenced).
    lib = dsa.load()
    p = dsa.make_problem(1, 8, 9_000_000, 8, 9_000_000, 64)
    fake = ctypes.c_void_p(1 << 20)
    args = [ctypes.byref(p), fake, None, fake, None, fake, fake, fake, fake, fake, fake, None]
    assert lib.dsa_forward_noalloc(*args) == 3   # DSA_ERR_WORKSPACE
