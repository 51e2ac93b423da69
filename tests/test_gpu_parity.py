"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs.  Tolerances are defined in gpu_utils.py and restated there.

Small sizes compare every element and span several tiles plus a ragged tail; the
full-size workloads compare sampled rows in the launch configuration bench.py times.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import attention_lightning_indexer_b200 as dsa
import dsa_synth
import oracle
from gpu_utils import (LSE_ATOL, O_ATOL, RECALL_MIN, assert_scores_close, fp8_to_f64, recall_excluding_near_ties,
                       sample_rows, score_bound_row, sorted_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCALE = dsa_synth.SM_SCALE


def _scores_buffer(rows: int, max_len_k: int, fill=float("nan")):
    return torch.full((rows, dsa.scores_ld(max_len_k)), fill, dtype=torch.float32, device=DEV)


def _cu(lens_q, lens_k):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    return cu_q, cu_k


# ------------------------------------------------------------------------- top-k

def _tie_heavy_scores(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    sc = torch.randn(rows, cols, generator=g).mul_(4).round_().div_(4)
    sc[torch.rand(rows, cols, generator=g) < 0.02] = -0.0
    sc[torch.rand(rows, cols, generator=g) < 0.02] = 0.0
    return sc


@pytest.mark.parametrize("L,k", [(256, 64), (700, 128), (5000, 2048), (3000, 1), (2100, 2048)])
def test_topk_bit_exact_on_identical_scores(L, k):
    sc = _tie_heavy_scores(L, L, seed=L + k)
    above = torch.triu(torch.ones(L, L, dtype=torch.bool), 1)
    sc = sc.masked_fill(above, 1e30)          # future entries: never read by either side
    sc_gpu = _scores_buffer(L, L)
    sc_gpu[:, :L] = sc.to(DEV)
    p = dsa.make_problem(1, L, L, L, L, k)
    idx = torch.full((L, k), -7, dtype=torch.int32, device=DEV)
    dsa.dsa_topk(p, sc_gpu, idx)
    ref = oracle.topk(sc_gpu[:, :L].cpu(), k)
    np.testing.assert_array_equal(sorted_rows(idx.cpu().numpy()), sorted_rows(ref))


def test_topk_long_rows_from_global_memory_and_ragged_batch():
    # Sequence 0 is longer than the shared-memory staging capacity; sequence 1 is short.
    lens_k = [60000, 1000]
    lens_q = [3, 3]
    cu_q, cu_k = _cu(lens_q, lens_k)
    k = 2048
    sc = _tie_heavy_scores(6, 60000, seed=5)
    sc_gpu = _scores_buffer(6, 60000, fill=0.0)
    sc_gpu[:, :60000] = sc.to(DEV)
    p = dsa.make_problem(2, 6, sum(lens_k), 3, 60000, k, cu_q=torch.from_numpy(cu_q).to(DEV),
                         cu_k=torch.from_numpy(cu_k).to(DEV))
    idx = torch.empty((6, k), dtype=torch.int32, device=DEV)
    dsa.dsa_topk(p, sc_gpu, idx)
    ref = oracle.topk(sc_gpu.cpu()[:, :60000], k, rows=np.arange(6), cu_q=cu_q, cu_k=cu_k)
    np.testing.assert_array_equal(sorted_rows(idx.cpu().numpy()), sorted_rows(ref))


@pytest.mark.parametrize("rows", [8, 200])
@pytest.mark.parametrize("pattern", ["constant", "increasing", "two_values", "spike"])
def test_topk_adversarial_rows_take_every_path(pattern, rows):
    # Rows built so that the sampled fast path is exact (spike), or must give up (all
    # keys equal; all top keys clustered in one warp's range; two values) and the general
    # path decides.  Either way the result must equal the oracle's.  8 rows run with
    # 1024 threads per row (fewer rows than SMs), 200 rows with 256.
    L, k = 6000, 2048
    base = torch.arange(L, dtype=torch.float32)
    if pattern == "constant":
        sc = torch.full((rows, L), 1.5)
    elif pattern == "increasing":
        sc = base.repeat(rows, 1) * 0.25
    elif pattern == "two_values":
        sc = (base.repeat(rows, 1) % 7 == 0).float() * 3.0 - 1.0
    else:
        sc = torch.randn(rows, L, generator=torch.Generator().manual_seed(3))
        sc[:, 100] = 1e6
    p = dsa.make_problem(1, L, L, L, L, k)
    buf = _scores_buffer(rows, L, fill=0.0)
    buf[:, :L] = sc.to(DEV)
    idx = torch.empty((rows, k), dtype=torch.int32, device=DEV)
    r0 = L - rows
    dsa.dsa_topk(p, buf, idx, row_begin=r0, row_count=rows)
    ref = oracle.topk(buf.cpu()[:, :L], k, rows=np.arange(r0, L), cu_q=[0, L], cu_k=[0, L])
    np.testing.assert_array_equal(sorted_rows(idx.cpu().numpy()), sorted_rows(ref))


def test_topk_row_subrange_and_empty_rows():
    L, k = 300, 32
    sc = _tie_heavy_scores(L, L, seed=9)
    sc_gpu = _scores_buffer(100, L, fill=0.0)
    sc_gpu[:, :L] = sc[150:250].to(DEV)
    p = dsa.make_problem(1, L, L, L, L, k)
    idx = torch.empty((100, k), dtype=torch.int32, device=DEV)
    dsa.dsa_topk(p, sc_gpu, idx, row_begin=150, row_count=100)
    ref = oracle.topk(sc_gpu.cpu()[:, :L], k, rows=np.arange(150, 250), cu_q=[0, L], cu_k=[0, L])
    np.testing.assert_array_equal(sorted_rows(idx.cpu().numpy()), sorted_rows(ref))
    dsa.dsa_topk(p, sc_gpu, idx, row_begin=0, row_count=0)   # empty launch is a no-op


# ----------------------------------------------------------------------- indexer

def _host_rows(t, rows):
    """Rows `rows` of a device tensor, gathered on the device and copied to the host (the
    full-size inputs are tens of GB; only the sampled rows travel)."""
    return t[torch.as_tensor(np.asarray(rows), device=t.device)].cpu()


def _scales(inp):
    """(q_scale, k_scale) device tensors of an FP8 input set (fp32 per token or ue8m0 blocks)."""
    if "q_scale_ue8m0" in inp:
        return inp["q_scale_ue8m0"], inp["k_scale_ue8m0"]
    return inp.get("q_scale"), inp.get("k_scale")


def _oracle_scores(inp, rows):
    cu_q = inp["cu_q"].cpu().numpy()
    cu_k = inp["cu_k"].cpu().numpy()
    if "q_scale_ue8m0" in inp:
        return oracle.indexer_fp8_block(_host_rows(inp["q_idx8"], rows), _host_rows(inp["q_scale_ue8m0"], rows),
                                        _host_rows(inp["w"], rows), inp["k_idx8"].cpu(), inp["k_scale_ue8m0"].cpu(),
                                        rows=rows, cu_q=cu_q, cu_k=cu_k, ld=inp["max_len_k"])
    if "q_idx8" in inp:
        qr = _host_rows(inp["q_idx8"], rows)
        qs = _host_rows(inp["q_scale"], rows)
        ref = oracle.indexer_fp8(qr, qs, _host_rows(inp["w"], rows), inp["k_idx8"].cpu(), inp["k_scale"].cpu(),
                                 rows=rows, cu_q=cu_q, cu_k=cu_k, ld=inp["max_len_k"])
        return ref
    return oracle.indexer(_host_rows(inp["q_idx"], rows), _host_rows(inp["w"], rows), inp["k_idx"].cpu(), rows=rows,
                          cu_q=cu_q, cu_k=cu_k, ld=inp["max_len_k"])


def _bound_rows(inp, rows):
    """Per listed row, the score tolerance scale of its visible keys 0..pos(t)."""
    pos = _positions(inp, rows)
    kb = _kbase(inp, rows)
    blocks = "q_scale_ue8m0" in inp
    if "q_idx8" in inp:
        q_sel = _host_rows(inp["q_idx8"], rows)
        if blocks:
            qs_sel = _host_rows(inp["q_scale_ue8m0"], rows).view(torch.float8_e8m0fnu).double()
            k_all = fp8_to_f64(inp["k_idx8"].cpu()) * inp["k_scale_ue8m0"].cpu().view(torch.float8_e8m0fnu).double()[:, None]
        else:
            qs_sel = _host_rows(inp["q_scale"], rows)
            k_all = fp8_to_f64(inp["k_idx8"].cpu()) * inp["k_scale"].cpu().double()[:, None]
    else:
        q_sel = _host_rows(inp["q_idx"], rows)
        k_all = inp["k_idx"].cpu()
    w_sel = _host_rows(inp["w"], rows)
    out = []
    for i, t in enumerate(rows):
        if "q_idx8" in inp and blocks:
            qr = fp8_to_f64(q_sel[i]) * qs_sel[i][:, None]
        elif "q_idx8" in inp:
            qr = fp8_to_f64(q_sel[i]) * float(qs_sel[i])
        else:
            qr = q_sel[i]
        n = int(pos[i]) + 1
        out.append(score_bound_row(qr, w_sel[i], k_all[int(kb[i]):int(kb[i]) + n]))
    return out


def _positions(inp, rows):
    return oracle.positions(rows, inp["cu_q"].cpu().numpy(), inp["cu_k"].cpu().numpy())


def _kbase(inp, rows):
    cu_q = inp["cu_q"].cpu().numpy()
    cu_k = inp["cu_k"].cpu().numpy()
    return np.array([cu_k[np.searchsorted(cu_q, t, side="right") - 1] for t in rows])


def _gpu_scores(inp, p):
    T = inp["total_q"]
    sc = _scores_buffer(T, inp["max_len_k"])
    if "q_idx8" in inp:
        qs, ks = _scales(inp)
        dsa.dsa_indexer_scores(p, inp["q_idx8"], inp["k_idx8"], inp["w"], sc, q_scale=qs, k_scale=ks)
    else:
        dsa.dsa_indexer_scores(p, inp["q_idx"], inp["k_idx"], inp["w"], sc)
    return sc


def _check_indexer(inp, rows):
    p = dsa.problem_from_inputs(inp)
    sc = _gpu_scores(inp, p).cpu().numpy()[rows]
    ref = _oracle_scores(inp, rows)
    pos = _positions(inp, rows)
    assert_scores_close(sc, ref, _bound_rows(inp, rows), pos)


@pytest.mark.parametrize("L,seed", [(256, 0), (700, 1), (1000, 2)])
def test_indexer_bf16_all_rows(L, seed):
    inp = dsa_synth.make_prefill(L, topk=64, seed=seed, device=DEV)
    _check_indexer(inp, np.arange(L))


def test_indexer_fp8_all_rows():
    inp = dsa_synth.make_prefill(700, topk=64, seed=3, device=DEV, fp8_indexer=True)
    _check_indexer(inp, np.arange(700))


def test_indexer_fp8_ue8m0_block_scales_all_rows():
    # e4m3 codes with power-of-two scales per 128-element block (per head of a query token,
    # per key token), given as ue8m0 bytes
    inp = dsa_synth.make_prefill(700, topk=64, seed=34, device=DEV, fp8_blocks=True)
    _check_indexer(inp, np.arange(700))


def test_forward_fp8_ue8m0_block_scales():
    inp = dsa_synth.make_prefill(5000, topk=512, seed=35, device=DEV, fp8_blocks=True)
    _check_forward_rows(inp, sample_rows(5000, 512, n_rand=24, seed=35, edge=6), chunk=1024)


def test_indexer_ragged_batch_several_queries_per_sequence():
    inp = dsa_synth.make_decode(5, 150, 900, topk=64, seed=4, device=DEV, q_per_seq=3)
    _check_indexer(inp, np.arange(inp["total_q"]))


# ---------------------------------------------------------------- sparse MLA

def _random_idx(inp, k, seed, sprinkle_invalid=True):
    rng = np.random.default_rng(seed)
    T = inp["total_q"]
    pos = _positions(inp, np.arange(T))
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = min(k, int(pos[t]) + 1)
        idx[t, :n] = rng.choice(int(pos[t]) + 1, n, replace=False)
        if sprinkle_invalid and n < k:
            idx[t, n] = int(pos[t]) + 1 + rng.integers(0, 5)   # future key: masked
            if n + 1 < k:
                idx[t, n + 1] = -3
        rng.shuffle(idx[t])
    return idx


def _check_mla(inp, idx_np, rows=None):
    T = inp["total_q"]
    p = dsa.problem_from_inputs(inp)
    idx = torch.from_numpy(idx_np).to(DEV)
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 128), dtype=torch.float32, device=DEV)
    dsa.dsa_sparse_mla_fwd(p, inp["q"], inp["kv"], idx, out, lse)
    rows = np.arange(T) if rows is None else rows
    rt = torch.from_numpy(rows)
    o_ref, lse_ref = oracle.sparse_mla(inp["q"].cpu()[rt], inp["kv"].cpu(), idx_np[rows], SCALE, rows=rows,
                                       cu_q=inp["cu_q"].cpu().numpy(), cu_k=inp["cu_k"].cpu().numpy())
    o = out.cpu()[rt].double().numpy()
    ls = lse.cpu()[rt].double().numpy()
    assert np.max(np.abs(o - o_ref)) <= O_ATOL
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(ls))
    assert np.max(np.abs(ls[fin] - lse_ref[fin]), initial=0.0) <= LSE_ATOL
    return out, lse


@pytest.mark.parametrize("L,k,std", [(256, 64, 1 / 24), (700, 128, 1.0), (300, 512, 1.0)])
def test_sparse_mla_same_index_set(L, k, std):
    inp = dsa_synth.make_prefill(L, topk=k, seed=L, device=DEV, latent_std=std)
    _check_mla(inp, _random_idx(inp, k, seed=L))


def test_sparse_mla_rows_without_valid_keys():
    inp = dsa_synth.make_prefill(64, topk=16, seed=11, device=DEV)
    idx = _random_idx(inp, 16, seed=11)
    idx[5] = -1
    idx[9] = 60       # all future for row 9 (pos 9) -> masked
    out, lse = _check_mla(inp, idx)
    assert torch.all(out[5] == 0) and torch.all(torch.isneginf(lse[5]))
    assert torch.all(out[9] == 0) and torch.all(torch.isneginf(lse[9]))


def test_sparse_mla_units_of_every_length_in_one_pair():
    # 600 rows on at most 74 CTA pairs: each pair walks ~8 rows in turn, among them rows
    # without a visible slot (all -1, or only future keys), rows whose only visible slot is
    # the first or the last one (1 or 4 blocks), and rows with holes; the pipeline state
    # carried from row to row must not leak into the next row's output
    L, k = 600, 1000
    inp = dsa_synth.make_prefill(L, topk=k, seed=21, device=DEV)
    idx = _random_idx(inp, k, seed=21)
    rng = np.random.default_rng(22)
    rows = rng.permutation(np.arange(100, L))
    empty, future, first, last, holes = np.split(rows[:250], 5)
    idx[empty] = -1
    for t in future:
        idx[t] = t + 1 + rng.integers(0, L - t - 1, k) if t + 2 < L else -1   # keys after pos(t) = t
    for t in first:
        idx[t] = -1
        idx[t, 0] = rng.integers(0, t + 1)
    for t in last:
        idx[t] = -1
        idx[t, k - 1] = rng.integers(0, t + 1)
    for t in holes:
        idx[t, rng.choice(k, k // 2, replace=False)] = -1
    out, lse = _check_mla(inp, idx)
    for t in np.concatenate([empty, future]):
        assert torch.all(out[int(t)] == 0) and torch.all(torch.isneginf(lse[int(t)]))


def test_sparse_mla_topk_not_multiple_of_four_with_repeated_indices():
    # 130 slots: rows of idx are not 16-byte aligned (scalar index loads) and the second
    # block is partial; some rows list a visible key twice (it counts once per occurrence)
    L, k = 400, 130
    inp = dsa_synth.make_prefill(L, topk=k, seed=13, device=DEV)
    idx = _random_idx(inp, k, seed=13)
    rng = np.random.default_rng(14)
    for t in rng.choice(np.arange(200, L), 40, replace=False):
        valid = np.nonzero((idx[t] >= 0) & (idx[t] <= t))[0]
        idx[t, valid[1]] = idx[t, valid[0]]
    _check_mla(inp, idx)


def test_empty_query_set_is_a_no_op():
    S, k = 300, 64
    p = dsa.make_problem(1, 0, S, 0, S, k)
    kv = torch.zeros((S, 576), dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((0, 128, 576), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((0, k), dtype=torch.int32, device=DEV)
    out = torch.zeros((0, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros((0, 128), dtype=torch.float32, device=DEV)
    dsa.dsa_sparse_mla_fwd(p, q, kv, idx, out, lse)
    ws = torch.empty(dsa.dsa_forward_workspace_size(p, 0), dtype=torch.uint8, device=DEV)
    qi = torch.zeros((0, 64, 128), dtype=torch.bfloat16, device=DEV)
    ki = torch.zeros((S, 128), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((0, 64), dtype=torch.float32, device=DEV)
    dsa.dsa_forward(p, qi, ki, w, q, kv, out, lse, ws, idx_out=idx)
    dsa.dsa_check_device_errors()


def test_sparse_mla_decode_ragged():
    inp = dsa_synth.make_decode(6, 300, 3000, topk=256, seed=12, device=DEV)
    _check_mla(inp, _random_idx(inp, 256, seed=12))


# ---------------------------------------------------------------- fused forward

def _run_forward(inp, chunk=0, want_idx=True):
    T = inp["total_q"]
    p = dsa.problem_from_inputs(inp)
    ws = torch.empty(dsa.dsa_forward_workspace_size(p, chunk), dtype=torch.uint8, device=DEV)
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 128), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, inp["topk"]), dtype=torch.int32, device=DEV) if want_idx else None
    fp8 = "q_idx8" in inp
    qs, ks = _scales(inp)
    dsa.dsa_forward(p, inp["q_idx8"] if fp8 else inp["q_idx"], inp["k_idx8"] if fp8 else inp["k_idx"], inp["w"],
                    inp["q"], inp["kv"], out, lse, ws, chunk_q=chunk, idx_out=idx, q_scale=qs, k_scale=ks)
    return idx, out, lse


def _check_forward_rows(inp, rows, chunk=0):
    idx, out, lse = _run_forward(inp, chunk)
    k = inp["topk"]
    pos = _positions(inp, rows)
    ref_sc = _oracle_scores(inp, rows)
    bound = _bound_rows(inp, rows)
    gidx = _host_rows(idx, rows).numpy()
    recall, wrong = recall_excluding_near_ties(gidx, ref_sc, bound, pos, k)
    assert recall >= RECALL_MIN and wrong == 0, (recall, wrong)
    o_ref, lse_ref = oracle.sparse_mla(_host_rows(inp["q"], rows), inp["kv"].cpu(), gidx, SCALE, rows=rows,
                                       cu_q=inp["cu_q"].cpu().numpy(), cu_k=inp["cu_k"].cpu().numpy())
    assert np.max(np.abs(_host_rows(out, rows).double().numpy() - o_ref)) <= O_ATOL
    assert np.max(np.abs(_host_rows(lse, rows).double().numpy() - lse_ref)) <= LSE_ATOL
    return idx, out, lse


def test_forward_ragged_batch_of_70_with_sequences_without_queries():
    # 70 sequences: more than one warp's worth of candidates, so each kernel's search over
    # cu_q takes two rounds; 0 to 6 queries per sequence, the first, last and the ones around
    # the warp boundary without any
    inp = dsa_synth.make_decode(70, 300, 3000, topk=256, seed=41, device=DEV, q_per_seq=6)
    rng = np.random.default_rng(41)
    qc = rng.integers(0, 7, 70)
    qc[[0, 5, 31, 32, 33, 69]] = 0
    T = int(qc.sum())
    for name in ("q_idx", "w", "q"):
        inp[name] = inp[name][:T].contiguous()
    inp["cu_q"] = torch.from_numpy(np.concatenate([[0], np.cumsum(qc)]).astype(np.int32)).to(DEV)
    inp["total_q"], inp["max_len_q"] = T, int(qc.max())
    _check_forward_rows(inp, np.arange(T))


def test_forward_pr_reference_config_all_rows():
    inp = dsa_synth.make_workload("pr_ref_256", seed=0, device=DEV)
    _check_forward_rows(inp, np.arange(256))


def test_forward_chunking_is_bit_identical():
    inp = dsa_synth.make_prefill(1000, topk=128, seed=21, device=DEV)
    a = _run_forward(inp, chunk=0)
    b = _run_forward(inp, chunk=96)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = _run_forward(inp, chunk=0, want_idx=False)
    assert torch.equal(a[1], c[1]) and torch.equal(a[2], c[2])


def test_forward_fp8_indexer_small():
    inp = dsa_synth.make_prefill(1200, topk=256, seed=22, device=DEV, fp8_indexer=True)
    _check_forward_rows(inp, sample_rows(1200, 256, n_rand=48, seed=22), chunk=512)


def test_forward_topk_not_multiple_of_four():
    inp = dsa_synth.make_prefill(600, topk=77, seed=24, device=DEV)
    _check_forward_rows(inp, np.arange(600), chunk=256)


def test_forward_decode_small_ragged():
    inp = dsa_synth.make_decode(6, 500, 5000, topk=512, seed=23, device=DEV)
    _check_forward_rows(inp, np.arange(6))


# ------------------------------------- split attention (few tokens: several CTA pairs each)

def test_forward_decode_batch_4_splits_each_row_over_8_pairs():
    # 4 tokens, index_topk 2048: each row's 8 blocks of 256 slots go to 8 CTA pairs whose
    # partial outputs are merged by their lse
    inp = dsa_synth.make_decode(4, 5000, 20000, topk=2048, seed=61, device=DEV)
    _, out, lse = _check_forward_rows(inp, np.arange(4))
    # the unsplit kernel on the same indices agrees to rounding
    p = dsa.problem_from_inputs(inp)
    idx = torch.empty((4, 2048), dtype=torch.int32, device=DEV)
    ws = torch.empty(dsa.dsa_forward_workspace_size(p, 0), dtype=torch.uint8, device=DEV)
    o2 = torch.empty_like(out)
    l2 = torch.empty_like(lse)
    dsa.dsa_forward(p, inp["q_idx"], inp["k_idx"], inp["w"], inp["q"], inp["kv"], o2, l2, ws, idx_out=idx)
    o1 = torch.empty_like(out)
    l1 = torch.empty_like(lse)
    dsa.dsa_sparse_mla_fwd(p, inp["q"], inp["kv"], idx, o1, l1)
    assert torch.max(torch.abs(o1.float() - o2.float())).item() <= 2e-2
    assert torch.max(torch.abs(l1 - l2)).item() <= 2e-3


def test_forward_decode_split_with_empty_parts():
    # contexts from 300 keys: a short row has fewer blocks than splits, so some of its parts
    # hold no visible slot (lse -inf, weight 0 in the merge)
    inp = dsa_synth.make_decode(6, 300, 9000, topk=2048, seed=62, device=DEV)
    lens = (inp["cu_k"][1:] - inp["cu_k"][:-1]).cpu().numpy()
    assert lens.min() < 7 * 256 and inp["max_len_k"] > 3584   # empty parts, and the gathered form
    _check_forward_rows(inp, np.arange(6))


def test_forward_decode_split_topk_512_three_queries_per_sequence():
    inp = dsa_synth.make_decode(3, 4000, 12000, topk=512, seed=63, device=DEV, q_per_seq=3)
    _check_forward_rows(inp, np.arange(9))


# ------------------------------------------- full-size workloads, sampled rows

def test_prefill_4k_full_size_sampled():
    inp = dsa_synth.make_workload("prefill_4k", seed=0, device=DEV)
    rows = sample_rows(4096, 2048, n_rand=24, seed=1, edge=8)
    _check_forward_rows(inp, rows, chunk=4096)


def test_forward_first_rows_take_the_dense_form_bit_identically():
    # one 5000-token sequence, index_topk 2048: rows 0..2047 see at most 2048 keys and
    # select all of them, so dsa_forward runs them in the dense form and the rest gathered;
    # the output equals the gathered form over the same indices bit for bit
    L, k = 5000, 2048
    inp = dsa_synth.make_prefill(L, topk=k, seed=34, device=DEV)
    idx, out, lse = _run_forward(inp)
    p = dsa.problem_from_inputs(inp)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    dsa.dsa_sparse_mla_fwd(p, inp["q"], inp["kv"], idx, out2, lse2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    _check_forward_rows(inp, np.array([0, 1, 1000, 2046, 2047, 2048, 2049, 4999]))


def test_prefill_3k_forward_takes_the_masked_dense_form():
    # topk < max_len_k <= the short-sequence threshold: dsa_forward runs the indexer and the
    # top-k, then the dense form restricted to the selected keys (its key blocks group the
    # keys differently from the gathered form, so the two agree to rounding, not bit for
    # bit); checked against the oracle on sampled rows
    inp = dsa_synth.make_workload("prefill_4k", seed=5, device=DEV, L=3072)
    _check_forward_rows(inp, sample_rows(3072, 2048, n_rand=12, seed=6, edge=4))


def test_prefill_32k_full_size_sampled_bench_config():
    inp = dsa_synth.make_workload("prefill_32k", seed=0, device=DEV)
    rows = sample_rows(32768, 2048, n_rand=12, seed=2, edge=4)
    _check_forward_rows(inp, rows, chunk=dsa_synth.WORKLOADS["prefill_32k"].chunk)


def test_prefill_128k_fp8_full_size_sampled_bench_config():
    # 131072 tokens, FP8 indexer with per-token scales, 4096-query chunks (the bench's launch
    # configuration); the oracle checks a handful of rows (each scores up to 128K keys)
    inp = dsa_synth.make_workload("prefill_128k_fp8", seed=0, device=DEV)
    rows = sample_rows(131072, 2048, n_rand=3, seed=4, edge=2)
    _check_forward_rows(inp, rows, chunk=dsa_synth.WORKLOADS["prefill_128k_fp8"].chunk)
    del inp
    torch.cuda.empty_cache()


def test_decode_b64_full_size_sampled():
    # every one of the 64 sequences: each seeded context length is covered
    inp = dsa_synth.make_workload("decode_b64", seed=0, device=DEV)
    _check_forward_rows(inp, np.arange(64))


# ------------------------------------------------------------ failure path

def test_bounded_wait_gives_up_reports_and_clears():
    # A one-CTA kernel waits ~1 ms on a barrier that nothing signals: the wait gives up
    # instead of hanging, the sticky flag reports DSA_ERR_DEVICE_TIMEOUT once, and the
    # device keeps working (a real forward right after is still exact).
    dsa.dsa_check_device_errors()                       # start from a clear flag
    dsa.dsa_selftest_bounded_wait(1000)
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_check_device_errors()
    assert e.value.code == 5
    dsa.dsa_check_device_errors()                       # cleared by the read
    inp = dsa_synth.make_workload("pr_ref_256", seed=0, device=DEV)
    _check_forward_rows(inp, np.arange(0, 256, 17))
    dsa.dsa_check_device_errors()


# ------------------------------------------------- dense (masked MHA) form

def _all_causal_idx(inp, k):
    """Index rows listing every visible key in order (what the top-k returns when pos + 1 <= k)."""
    T = inp["total_q"]
    pos = _positions(inp, np.arange(T))
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = min(k, int(pos[t]) + 1)
        idx[t, :n] = np.arange(n)
    return idx


def _oracle_mla(inp, idx_np):
    return oracle.sparse_mla(inp["q"].cpu(), inp["kv"].cpu(), idx_np, SCALE, rows=np.arange(inp["total_q"]),
                             cu_q=inp["cu_q"].cpu().numpy(), cu_k=inp["cu_k"].cpu().numpy())


def _assert_mla_close(out, lse, o_ref, lse_ref):
    assert np.max(np.abs(out.cpu().double().numpy() - o_ref)) <= O_ATOL
    ls = lse.cpu().double().numpy()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(ls))
    assert np.max(np.abs(ls[fin] - lse_ref[fin]), initial=0.0) <= LSE_ATOL


@pytest.mark.parametrize("L,std", [(300, 1.0), (700, 1 / 24)])
def test_dense_mla_over_all_causal_keys(L, std):
    # idx = NULL: every key 0..pos(t) attends -- the oracle's sparse attention over index rows
    # listing all causal keys (which the pins tie to textbook dense causal attention)
    inp = dsa_synth.make_prefill(L, topk=L, seed=L + 1, device=DEV, latent_std=std)
    p = dsa.problem_from_inputs(inp)
    out = torch.empty((L, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((L, 128), dtype=torch.float32, device=DEV)
    dsa.dsa_dense_mla_fwd(p, inp["q"], inp["kv"], None, out, lse)
    _assert_mla_close(out, lse, *_oracle_mla(inp, _all_causal_idx(inp, L)))


def test_dense_mla_masked_by_index_rows_equals_sparse_attention():
    # index rows with distinct keys plus ignored entries (a future key, -3): the dense form
    # restricted to them computes the same attention as the gathered form
    L, k = 1000, 128
    inp = dsa_synth.make_prefill(L, topk=k, seed=31, device=DEV)
    idx_np = _random_idx(inp, k, seed=31)
    p = dsa.problem_from_inputs(inp)
    out = torch.empty((L, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((L, 128), dtype=torch.float32, device=DEV)
    dsa.dsa_dense_mla_fwd(p, inp["q"], inp["kv"], torch.from_numpy(idx_np).to(DEV), out, lse)
    _assert_mla_close(out, lse, *_oracle_mla(inp, idx_np))


def test_dense_mla_masked_rows_without_listed_keys_among_others():
    # 500 rows walked by at most 74 pairs; some index rows list no visible key (all -1, or
    # only keys after pos(t)): those rows still run their blocks (the dense form's blocks come
    # from pos(t)) and must come out as 0 / -inf, and the next row of the pair must not see
    # their state
    L, k = 500, 96
    inp = dsa_synth.make_prefill(L, topk=k, seed=33, device=DEV)
    idx_np = _random_idx(inp, k, seed=33)
    rng = np.random.default_rng(34)
    rows = rng.choice(np.arange(50, L - 2), 60, replace=False)
    idx_np[rows[:30]] = -1
    for t in rows[30:]:
        idx_np[t] = t + 1 + rng.integers(0, L - t - 1, k)
    p = dsa.problem_from_inputs(inp)
    out = torch.empty((L, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((L, 128), dtype=torch.float32, device=DEV)
    dsa.dsa_dense_mla_fwd(p, inp["q"], inp["kv"], torch.from_numpy(idx_np).to(DEV), out, lse)
    _assert_mla_close(out, lse, *_oracle_mla(inp, idx_np))
    for t in rows:
        assert torch.all(out[int(t)] == 0) and torch.all(torch.isneginf(lse[int(t)]))


def test_dense_mla_ragged_decode_masked():
    inp = dsa_synth.make_decode(5, 300, 3000, topk=256, seed=32, device=DEV)
    idx_np = _random_idx(inp, 256, seed=32)
    T = inp["total_q"]
    p = dsa.problem_from_inputs(inp)
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, 128), dtype=torch.float32, device=DEV)
    dsa.dsa_dense_mla_fwd(p, inp["q"], inp["kv"], torch.from_numpy(idx_np).to(DEV), out, lse)
    _assert_mla_close(out, lse, *_oracle_mla(inp, idx_np))


def test_forward_short_sequence_takes_the_dense_path_bit_identically():
    # max_len_k <= topk: every visible key is selected, so dsa_forward skips the indexer and
    # the top-k; the result must equal the explicit indexer -> top-k -> gathered path bit for bit
    L, k = 200, 256
    inp = dsa_synth.make_prefill(L, topk=k, seed=33, device=DEV)
    idx_f, out_f, lse_f = _run_forward(inp)
    p = dsa.problem_from_inputs(inp)
    sc = _gpu_scores(inp, p)
    idx = torch.empty((L, k), dtype=torch.int32, device=DEV)
    dsa.dsa_topk(p, sc, idx)
    out = torch.empty_like(out_f)
    lse = torch.empty_like(lse_f)
    dsa.dsa_sparse_mla_fwd(p, inp["q"], inp["kv"], idx, out, lse)
    assert torch.equal(idx_f, idx)
    assert torch.equal(out_f, out) and torch.equal(lse_f, lse)
    np.testing.assert_array_equal(idx.cpu().numpy(), _all_causal_idx(inp, k))
    _check_forward_rows(inp, np.arange(0, L, 7))


# ------------------------------------------------------- paged key caches

def _paged(inp, seed):
    pg = dsa_synth.to_paged(inp, page_size=64, seed=seed)
    assert pg["block_table"].device.type == "cuda"
    return pg


@pytest.mark.parametrize("fp8", [False, True])
def test_indexer_paged_cache_equals_packed(fp8):
    inp = dsa_synth.make_decode(5, 150, 1500, topk=64, seed=51, device=DEV, q_per_seq=3)
    if fp8:
        q8, qs = dsa_synth.quantize_e4m3_per_token(inp["q_idx"].float())
        k8, ks = dsa_synth.quantize_e4m3_per_token(inp["k_idx"].float())
        inp = {kk: v for kk, v in inp.items() if kk not in ("q_idx", "k_idx")}
        inp.update(q_idx8=q8, q_scale=qs, k_idx8=k8, k_scale=ks)
    pg = _paged(inp, seed=52)
    a = _gpu_scores(inp, dsa.problem_from_inputs(inp))
    b = _gpu_scores(pg, dsa.problem_from_inputs(pg))
    rows = np.arange(inp["total_q"])
    pos = _positions(inp, rows)
    for r in rows:
        n = int(pos[r]) + 1
        assert torch.equal(a[r, :n], b[r, :n])


def _forward_paged_vs_packed(inp, seed, rows):
    pg = _paged(inp, seed)
    idx_a, out_a, lse_a = _run_forward(inp)
    idx_b, out_b, lse_b = _run_forward(pg)
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)
    # and against the oracle reading the paged layout through the same block table
    cu_q = pg["cu_q"].cpu().numpy()
    cu_k = pg["cu_k"].cpu().numpy()
    table = pg["block_table"].cpu().numpy()
    gidx = _host_rows(idx_b, rows).numpy()
    o_ref, lse_ref = oracle.sparse_mla(_host_rows(pg["q"], rows), pg["kv"].cpu(), gidx, SCALE, rows=rows, cu_q=cu_q,
                                       cu_k=cu_k, block_table=table)
    assert np.max(np.abs(_host_rows(out_b, rows).double().numpy() - o_ref)) <= O_ATOL
    assert np.max(np.abs(_host_rows(lse_b, rows).double().numpy() - lse_ref)) <= LSE_ATOL
    sc_ref = oracle.indexer(_host_rows(pg["q_idx"], rows), _host_rows(pg["w"], rows), pg["k_idx"].cpu(), rows=rows,
                            cu_q=cu_q, cu_k=cu_k, ld=pg["max_len_k"], block_table=table)
    bound = _bound_rows(inp, rows)
    recall, wrong = recall_excluding_near_ties(gidx, sc_ref, bound, _positions(inp, rows), inp["topk"])
    assert recall >= RECALL_MIN and wrong == 0, (recall, wrong)


def test_forward_paged_decode_small():
    inp = dsa_synth.make_decode(6, 500, 5000, topk=512, seed=53, device=DEV)
    _forward_paged_vs_packed(inp, seed=54, rows=np.arange(6))


def test_forward_paged_decode_batch_4_split_attention():
    # 4 tokens: the attention splits each row over 8 CTA pairs and gathers through the table
    inp = dsa_synth.make_decode(4, 5000, 20000, topk=2048, seed=56, device=DEV)
    _forward_paged_vs_packed(inp, seed=57, rows=np.arange(4))


def test_forward_paged_decode_b64_full_size():
    inp = dsa_synth.make_workload("decode_b64", seed=0, device=DEV)
    _forward_paged_vs_packed(inp, seed=55, rows=np.array([0, 17, 40, 63]))


# ------------------------------------------------------ key-cache write producer

def test_cache_write_rows_against_oracle():
    # new tokens at positions up to 163,839 written to scattered cache rows (as through a
    # block table); rows that are not written keep their sentinel; tolerance: one bf16
    # rounding (2^-9 relative) of an fp32 computation, doubled
    n, cap = 777, 4096
    g = torch.Generator(device=DEV).manual_seed(81)
    k_raw = (torch.randn(n, 128, generator=g, device=DEV) * 2 + 0.5).to(torch.bfloat16)
    kv_raw = torch.randn(n, 576, generator=g, device=DEV).to(torch.bfloat16)
    pos = torch.randint(0, 163840, (n,), generator=g, device=DEV, dtype=torch.int32)
    pos[:3] = torch.tensor([0, 1, 163839], dtype=torch.int32, device=DEV)
    rows = torch.randperm(cap, generator=g, device=DEV)[:n].to(torch.int32)
    ln_w = torch.rand(128, generator=g, device=DEV) + 0.5
    ln_b = torch.randn(128, generator=g, device=DEV) * 0.1
    rms_w = torch.rand(512, generator=g, device=DEV) + 0.5
    inv_freq = torch.rand(32, generator=g, device=DEV) * 0.9 + 0.01
    kc = torch.full((cap, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    kvc = torch.full((cap, 576), 7.0, dtype=torch.bfloat16, device=DEV)
    dsa.dsa_cache_write(k_raw, kv_raw, pos, rows, ln_w, ln_b, rms_w, inv_freq, kc, kvc, eps=1e-6)
    ref_k, ref_kv = oracle.cache_write(k_raw.cpu(), kv_raw.cpu(), pos.cpu(), ln_w.cpu(), ln_b.cpu(), rms_w.cpu(),
                                       inv_freq.cpu(), 1e-6)
    r = rows.long().cpu()
    got_k = kc.cpu()[r].double().numpy()
    got_kv = kvc.cpu()[r].double().numpy()
    assert np.all(np.abs(got_k - ref_k) <= 2.0 ** -8 * np.abs(ref_k) + 1e-4)
    assert np.all(np.abs(got_kv - ref_kv) <= 2.0 ** -8 * np.abs(ref_kv) + 1e-4)
    untouched = np.setdiff1d(np.arange(cap), r.numpy())
    assert torch.all(kc.cpu()[untouched] == 7.0) and torch.all(kvc.cpu()[untouched] == 7.0)


# ------------------------------------------------------------ debug checks

def test_debug_checks_flag_and_skip_an_inconsistent_sequence():
    # The last sequence's key range runs 64 rows past total_k (its length stays within
    # max_len_k, so even unchecked every access would stay inside the buffers: TMA loads
    # past the arrays read zeros).  With debug checks on, that row is flagged and skipped
    # (no keys: idx -1, out 0, lse -inf) while the other rows are unchanged.
    inp = dsa_synth.make_decode(4, 5000, 6000, topk=256, seed=91, device=DEV)
    ref = _run_forward(inp)
    dsa.dsa_check_device_errors()
    bad = dict(inp)
    cu_k = inp["cu_k"].clone()
    cu_k[-1] += 64                                       # only the last sequence grows
    bad["cu_k"] = cu_k
    bad["max_len_k"] = inp["max_len_k"] + 64
    dsa.dsa_set_debug_checks(True)
    try:
        idx, out, lse = _run_forward(bad)
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_check_device_errors()
        assert e.value.code == 6
        dsa.dsa_check_device_errors()                    # cleared by the read
        assert torch.equal(idx[:3], ref[0][:3]) and torch.equal(out[:3], ref[1][:3]) and torch.equal(lse[:3], ref[2][:3])
        assert torch.all(idx[3] == -1) and torch.all(out[3] == 0) and torch.all(torch.isneginf(lse[3]))
        _run_forward(inp)                                # a consistent problem passes the checks
        dsa.dsa_check_device_errors()
        # FP8 with an fp32 scale that is not > 0
        f8 = dsa_synth.make_prefill(600, topk=64, seed=92, device=DEV, fp8_indexer=True)
        f8["k_scale"][17] = 0.0
        _gpu_scores(f8, dsa.problem_from_inputs(f8))
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_check_device_errors()
        assert e.value.code == 6
    finally:
        dsa.dsa_set_debug_checks(False)
        dsa.dsa_check_device_errors()
