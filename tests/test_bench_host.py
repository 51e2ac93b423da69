"""Host-side logic of bench.py on CPU: the replica plumbing under a 2-rank gloo process
group (barrier, max over ranks, the reference arm's rank-0-only rule) and the workload
bookkeeping behind the roofline figures (causal pairs, selected pairs, top-k bytes)."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    got_ws, got_rank, got_local = bench._dist()
    dist = bench._init_pg(got_ws, got_local, backend="gloo")
    try:
        bench._barrier(dist)
        mx = bench._max_over_ranks(dist, 10.0 + 3.0 * rank)       # per-rank "elapsed ms"
        bench._barrier(dist)
        out[rank] = (got_ws, got_rank, mx)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_barrier_and_max_over_ranks():
    ws = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(ws, _free_port(), out), nprocs=ws, start_method="spawn", join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank, (got_ws, got_rank, mx) in res.items():
        assert got_ws == ws and got_rank == rank
        assert mx == 13.0                                        # every rank sees the slowest rank's time


def test_single_process_helpers_are_identity():
    assert bench._init_pg(1, 0) is None
    bench._barrier(None)
    assert bench._max_over_ranks(None, 4.25) == 4.25


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        workload = "pr_ref_256"
        seed = 0
        cpu_rows = 4
        steps = 1
        warmup = 0
    bench.run_reference(Args(), ws=2, rank=1, local=1)           # a non-zero rank exits without work
    assert capsys.readouterr().out == ""


def _inp(cu_q, cu_k, topk):
    return {"cu_q": torch.tensor(cu_q, dtype=torch.int32), "cu_k": torch.tensor(cu_k, dtype=torch.int32), "topk": topk}


@pytest.mark.parametrize("L,k", [(7, 3), (256, 64), (300, 512)])
def test_pair_counts_prefill_match_brute_force(L, k):
    idx_pairs, mla_pairs, topk_bytes = bench._pairs(_inp([0, L], [0, L], k))
    vis = [t + 1 for t in range(L)]                              # keys 0..t visible to query t
    assert idx_pairs == sum(vis)
    assert mla_pairs == sum(min(n, k) for n in vis)
    assert topk_bytes == sum(4 * n for n in vis if n > k) + 4 * k * L


def test_pair_counts_ragged_decode_use_last_token_positions():
    # two sequences, 1 and 3 queries, contexts 10 and 6: queries sit at the end
    cu_q, cu_k, k = [0, 1, 4], [0, 10, 16], 4
    idx_pairs, mla_pairs, _ = bench._pairs(_inp(cu_q, cu_k, k))
    vis = [10] + [4, 5, 6]
    assert idx_pairs == sum(vis)
    assert mla_pairs == sum(min(n, k) for n in vis)


def test_metric_and_flop_constants_match_the_problem_shapes():
    assert bench.FLOP_PER_PAIR_INDEXER == 64 * 128 * 2
    assert bench.FLOP_PER_PAIR_MLA == 128 * (576 + 512) * 2
    assert "32K prefill" in bench.METRIC and "decode" in bench.METRIC
    assert np.isclose(bench.L2_BYTES, 126 * 2 ** 20)


def test_attention_launch_count_follows_the_forward_forms():
    # the forward's attention: the dense form alone up to the short-sequence threshold; in
    # one packed sequence the rows that see at most topk keys take the dense form and the
    # rest the gathered form (two launches); ragged or paged problems take one launch
    import attention_lightning_indexer_b200 as dsa
    assert bench._attention_launches(dsa.make_problem(1, 2048, 2048, 2048, 2048, 2048)) == 1
    assert bench._attention_launches(dsa.make_problem(1, 3584, 3584, 3584, 3584, 2048)) == 1
    assert bench._attention_launches(dsa.make_problem(1, 32768, 32768, 32768, 32768, 2048)) == 2
    # every row sees more than topk keys: gathered only
    assert bench._attention_launches(dsa.make_problem(1, 512, 40000, 512, 40000, 2048)) == 1
    # every row sees at most topk keys (but the sequence is longer than the threshold)
    assert bench._attention_launches(dsa.make_problem(1, 4000, 4000, 4000, 4000, 8192)) == 1


def test_workload_config_names_the_workload_and_its_launch_shape():
    # one helper builds the config of both arms (ours and --impl reference)
    import argparse
    args = argparse.Namespace(workload="prefill_32k")
    cfg = bench._config(args, {"batch": 1, "max_len_k": 32768, "topk": 2048}, 8192, 2)
    assert (cfg["workload"], cfg["global_batch"], cfg["seq_len"], cfg["topk"], cfg["chunk_q"]) == \
        ("prefill_32k", 2, 32768, 2048, 8192)
    assert cfg["parallelism"] == "replicas x2" and "l2" in cfg
