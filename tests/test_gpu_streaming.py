"""Streaming indexer -> top-k (no score rows) against the two-pass kernels, on a B200.

The streaming path must write exactly what dsa_indexer_scores followed by dsa_topk
writes: the same indices in the same slots, for every row, whatever its candidate
threshold did.  The cases below reach each way a row can go: decided from its
candidates, decided among tied candidates by index, and redone from full scores after
its threshold let too many (overflow) or too few keys through.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import attention_lightning_indexer_b200 as dsa
import dsa_synth
from gpu_utils import sorted_rows
from test_gpu_parity import _gpu_scores, _scales

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _two_pass(inp, p):
    sc = _gpu_scores(inp, p)
    idx = torch.empty((inp["total_q"], inp["topk"]), dtype=torch.int32, device=DEV)
    dsa.dsa_topk(p, sc, idx)
    return idx


def _streaming(inp, p, chunk=0, row_begin=0, row_count=None):
    T = inp["total_q"]
    n = T - row_begin if row_count is None else row_count
    ws = torch.empty(dsa.dsa_indexer_topk_streaming_workspace_size(p, chunk), dtype=torch.uint8, device=DEV)
    idx = torch.full((n, inp["topk"]), -7, dtype=torch.int32, device=DEV)
    fp8 = "q_idx8" in inp
    qs, ks = _scales(inp)
    dsa.dsa_indexer_topk_streaming(p, inp["q_idx8"] if fp8 else inp["q_idx"], inp["k_idx8"] if fp8 else inp["k_idx"],
                                   inp["w"], idx, ws, row_begin=row_begin, row_count=n, chunk_q=chunk, q_scale=qs,
                                   k_scale=ks)
    dsa.dsa_check_device_errors()
    return idx


@pytest.mark.parametrize("L,k,chunk", [(5000, 256, 0), (5000, 256, 768), (6000, 2048, 2048)])
def test_streaming_equals_two_pass(L, k, chunk):
    inp = dsa_synth.make_prefill(L, topk=k, seed=51, device=DEV, with_latent=False)
    p = dsa.problem_from_inputs(inp)
    assert torch.equal(_streaming(inp, p, chunk), _two_pass(inp, p))


def test_streaming_row_subrange():
    inp = dsa_synth.make_prefill(4000, topk=128, seed=52, device=DEV, with_latent=False)
    p = dsa.problem_from_inputs(inp)
    ref = _two_pass(inp, p)
    assert torch.equal(_streaming(inp, p, chunk=300, row_begin=1111, row_count=2222), ref[1111:3333])


@pytest.mark.parametrize("blocks", [False, True])
def test_streaming_fp8_equals_two_pass(blocks):
    inp = dsa_synth.make_prefill(4500, topk=512, seed=53, device=DEV, fp8_indexer=True, fp8_blocks=blocks,
                                 with_latent=False)
    p = dsa.problem_from_inputs(inp)
    assert torch.equal(_streaming(inp, p, chunk=1000), _two_pass(inp, p))


def test_streaming_all_tied_rows_take_index_order_and_overflow_is_redone():
    # w = 0: every score is 0.  Rows with at most 7168 keys keep all keys as candidates and
    # pick the k smallest indices among the ties; longer rows overflow the candidate list
    # and are redone from full scores
    inp = dsa_synth.make_prefill(9000, topk=256, seed=54, device=DEV, with_latent=False)
    inp["w"].zero_()
    p = dsa.problem_from_inputs(inp)
    got = _streaming(inp, p, chunk=4096)
    assert torch.equal(got, _two_pass(inp, p))
    want = np.tile(np.arange(256, dtype=np.int32), (9000, 1))
    want[:256] = -1
    for t in range(256):
        want[t, : t + 1] = np.arange(t + 1)
    np.testing.assert_array_equal(sorted_rows(got.cpu().numpy()), sorted_rows(want))


def test_streaming_misjudged_threshold_is_redone():
    # the sampled tiles (every 32nd tile of 128 keys) get keys 8x larger than the rest, so
    # the sample sets the threshold far too high and fewer than k keys reach it
    L, k = 8192, 1024
    inp = dsa_synth.make_prefill(L, topk=k, seed=55, device=DEV, with_latent=False)
    kk = inp["k_idx"].float()
    for j in range(0, L, 32 * 128):
        kk[j:j + 128] *= 8.0
    inp["k_idx"] = kk.to(torch.bfloat16)
    p = dsa.problem_from_inputs(inp)
    assert torch.equal(_streaming(inp, p, chunk=2048), _two_pass(inp, p))


def test_streaming_ragged_batch_uses_the_two_pass_kernels():
    inp = dsa_synth.make_decode(6, 3000, 9000, topk=512, seed=56, device=DEV, q_per_seq=3)
    p = dsa.problem_from_inputs(inp)
    assert torch.equal(_streaming(inp, p), _two_pass(inp, p))


def test_streaming_prefill_32k_full_size_every_row():
    # the headline workload in its launch configuration (8192-query chunks)
    inp = dsa_synth.make_workload("prefill_32k", seed=0, device=DEV, with_latent=False)
    p = dsa.problem_from_inputs(inp)
    got = _streaming(inp, p, chunk=dsa_synth.WORKLOADS["prefill_32k"].chunk)
    ch = dsa_synth.WORKLOADS["prefill_32k"].chunk
    T, ld = inp["total_q"], dsa.scores_ld(inp["max_len_k"])
    sc = torch.empty((ch, ld), dtype=torch.float32, device=DEV)
    ref = torch.empty_like(got)
    for r0 in range(0, T, ch):
        dsa.dsa_indexer_scores(p, inp["q_idx"], inp["k_idx"], inp["w"], sc, row_begin=r0, row_count=ch)
        dsa.dsa_topk(p, sc, ref[r0:r0 + ch], row_begin=r0, row_count=ch)
    assert torch.equal(got, ref)
