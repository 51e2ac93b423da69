"""Pins for the fp64 oracle: each test ties an oracle function to something other than
itself -- hand-worked values from the pages' definitions (tests/golden), closed forms,
invariants, special cases that reduce to a library routine, and brute force on tiny
inputs.  Chosen so that a dropped term, a wrong sign or index, a missing ReLU, a wrong
mask or a transposed operand fails at least one of them.

Page citations: "DeepSeek-V3.2 tech report summary" section 1 DSA (lightning indexer
formula, top-k selection, MQA-mode MLA); "Model techniques map -- DeepSeek-V3.2",
feature "Indexer-selected sparse attention" (topk = min(index_topk, len), int32).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ indexer pins

def test_indexer_hand_worked_tiny():
    g = _gold("indexer_tiny.json")
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    w = np.array(g["w"], dtype=np.float64)
    got = oracle.indexer(q, w, k)
    exp = np.array([[np.nan if v is None else v for v in row] for row in g["scores"]])
    for t in range(3):
        for s in range(3):
            if np.isnan(exp[t, s]):
                assert got[t, s] == -np.inf
            else:
                assert got[t, s] == exp[t, s]


def test_indexer_single_head_unit_weight_is_relu_matmul():
    # H_I = 1, w = 1: I = ReLU(Q K^T) on the causal triangle (numpy matmul + clip).
    r = _rng(1)
    L, D = 37, 16
    q = r.standard_normal((L, 1, D))
    k = r.standard_normal((L, D))
    w = np.ones((L, 1))
    got = oracle.indexer(q, w, k)
    ref = np.clip(q[:, 0, :] @ k.T, 0.0, None)
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(got[tri], ref[tri], rtol=1e-13, atol=1e-13)
    assert np.all(got[~tri] == -np.inf)


def test_indexer_relu_closed_form_under_key_negation():
    # relu(x) - relu(-x) = x, so I(q,k) - I(q,-k) = sum_j w[t,j] (q[t,j].k[s]).
    # Fails if the ReLU is dropped (difference doubles) or applied after the w-product.
    r = _rng(2)
    L, H, D = 29, 5, 12
    q = r.standard_normal((L, H, D))
    k = r.standard_normal((L, D))
    w = r.standard_normal((L, H))
    with np.errstate(invalid="ignore"):
        diff = oracle.indexer(q, w, k) - oracle.indexer(q, w, -k)
    lin = np.einsum("th,thd,sd->ts", w, q, k)
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(diff[tri], lin[tri], rtol=1e-12, atol=1e-12)


def test_indexer_linear_in_w_and_zero_heads_drop_out():
    r = _rng(3)
    L, H, D = 23, 6, 8
    q = r.standard_normal((L, H, D))
    k = r.standard_normal((L, D))
    w1 = r.standard_normal((L, H))
    w2 = r.standard_normal((L, H))
    tri = np.tril(np.ones((L, L), dtype=bool))
    a = oracle.indexer(q, w1 + 2.0 * w2, k)
    b = oracle.indexer(q, w1, k) + 2.0 * oracle.indexer(q, w2, k)
    np.testing.assert_allclose(a[tri], b[tri], rtol=1e-12, atol=1e-12)
    # Heads with zero weight contribute nothing: same as removing them.
    w3 = w1.copy()
    w3[:, [1, 4]] = 0.0
    keep = [0, 2, 3, 5]
    c = oracle.indexer(q, w3, k)
    d = oracle.indexer(q[:, keep, :], w1[:, keep], k)
    np.testing.assert_allclose(c[tri], d[tri], rtol=1e-12, atol=1e-12)


def test_indexer_positive_homogeneity_rows_and_columns():
    r = _rng(4)
    L, H, D = 19, 4, 8
    q = r.standard_normal((L, H, D))
    k = r.standard_normal((L, D))
    w = r.standard_normal((L, H))
    base = oracle.indexer(q, w, k)
    a = np.exp(r.standard_normal(L))          # per-query factor > 0
    b = np.exp(r.standard_normal(L))          # per-key factor > 0
    scaled = oracle.indexer(q * a[:, None, None], w, k * b[:, None])
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(scaled[tri], (base * a[:, None] * b[None, :])[tri], rtol=1e-12, atol=1e-12)


def test_indexer_ragged_batch_uses_own_keys_and_last_token_positions():
    # Two sequences; queries are the last tokens of each sequence.  Each row equals
    # the corresponding row of a standalone prefill of its own sequence, and keys of
    # the other sequence never enter.
    r = _rng(5)
    H, D = 3, 8
    lk = [11, 7]
    lq = [4, 7]
    k = r.standard_normal((sum(lk), D))
    q = r.standard_normal((sum(lq), H, D))
    w = r.standard_normal((sum(lq), H))
    cu_q = np.array([0, 4, 11], dtype=np.int32)
    cu_k = np.array([0, 11, 18], dtype=np.int32)
    got = oracle.indexer(q, w, k, cu_q=cu_q, cu_k=cu_k)
    assert got.shape == (11, 11)
    # sequence 0: standalone prefill of 11 tokens, rows 7..10
    q0 = np.concatenate([r.standard_normal((7, H, D)), q[:4]])
    w0 = np.concatenate([r.standard_normal((7, H)), w[:4]])
    ref0 = oracle.indexer(q0, w0, k[:11])
    np.testing.assert_array_equal(got[:4], ref0[7:])
    ref1 = oracle.indexer(q[4:], w[4:], k[11:])
    np.testing.assert_array_equal(got[4:, :7], ref1)
    assert np.all(got[4:, 7:] == -np.inf)


def test_positions_hand_worked_ragged_and_match_the_indexer_extent():
    # The boundary's ragged reading: the queries of sequence b are its last len_q(b)
    # tokens.  cu_q = [0, 4, 11], cu_k = [0, 11, 18]: sequence 0 has 11 keys and its 4
    # queries sit at positions 7..10; sequence 1 has 7 keys and 7 queries at 0..6.
    cu_q = np.array([0, 4, 11], dtype=np.int32)
    cu_k = np.array([0, 11, 18], dtype=np.int32)
    pos = oracle.positions(np.arange(11), cu_q, cu_k)
    np.testing.assert_array_equal(pos, [7, 8, 9, 10, 0, 1, 2, 3, 4, 5, 6])
    # The same positions, read off the C indexer: the last finite column of each row is
    # pos(t) (w > 0 and q = k = 1 make every visible score positive).
    H, D = 2, 4
    q = np.ones((11, H, D))
    k = np.ones((18, D))
    w = np.ones((11, H))
    sc = oracle.indexer(q, w, k, cu_q=cu_q, cu_k=cu_k)
    last = np.array([np.nonzero(np.isfinite(row))[0].max() for row in sc])
    np.testing.assert_array_equal(last, pos)
    # plain prefill (cu arrays of one sequence, T = L) and a decode batch (one query each)
    np.testing.assert_array_equal(oracle.positions(np.arange(5), [0, 5], [0, 5]), np.arange(5))
    np.testing.assert_array_equal(oracle.positions(np.arange(3), [0, 1, 2, 3], [0, 9, 10, 40]), [8, 0, 29])
    # queries that are the last 3 tokens of a 10-token prefix
    np.testing.assert_array_equal(oracle.positions(np.arange(3), [0, 3], [0, 10]), [7, 8, 9])


def test_e4m3_decoder_matches_library_cast():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if np.isnan(lib[c]):
            assert math.isnan(v)
        else:
            assert v == lib[c], (c, v, lib[c])
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9


def test_indexer_fp8_equals_float_indexer_on_dequantised_inputs():
    r = _rng(6)
    L, H, D = 17, 4, 16
    q8 = torch.from_numpy(r.integers(0, 256, (L, H, D), dtype=np.uint8))
    k8 = torch.from_numpy(r.integers(0, 256, (L, D), dtype=np.uint8))
    q8[(q8 & 0x7F) == 0x7F] = 0x10   # no NaN codes
    k8[(k8 & 0x7F) == 0x7F] = 0x22
    qs = np.exp(r.standard_normal(L))
    ks = np.exp(r.standard_normal(L))
    w = r.standard_normal((L, H))
    got = oracle.indexer_fp8(q8, qs, w, k8, ks)
    qf = q8.view(torch.float8_e4m3fn).to(torch.float64).numpy() * qs[:, None, None]
    kf = k8.view(torch.float8_e4m3fn).to(torch.float64).numpy() * ks[:, None]
    ref = oracle.indexer(qf, w, kf)
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(got[tri], ref[tri], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ top-k pins

def _brute_topk(row, pos, k):
    cand = list(range(pos + 1))
    cand.sort(key=lambda s: (-float(row[s]), s))
    sel = cand[:k]
    return sel + [-1] * (k - len(sel))


def test_topk_hand_worked_tiny():
    g = _gold("indexer_tiny.json")
    sc = np.array([[-np.inf if v is None else v for v in row] for row in g["scores"]])
    assert oracle.topk(sc, 2).tolist() == g["top2"]
    assert oracle.topk(sc, 1).tolist() == g["top1"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_brute_force_tiny(seed):
    r = _rng(10 + seed)
    L = 40
    sc = np.round(r.standard_normal((L, L)) * 3) / 2   # many ties on purpose
    sc = sc.astype(np.float32)
    for k in (1, 5, 16, 39, 40, 64):
        got = oracle.topk(sc, k)
        for t in range(L):
            assert got[t].tolist() == _brute_topk(sc[t], t, k), (k, t)


def test_topk_select_all_when_k_covers_prefix_and_padding_count():
    r = _rng(20)
    L, k = 50, 20
    sc = r.standard_normal((L, L)).astype(np.float32)
    got = oracle.topk(sc, k)
    for t in range(L):
        keff = min(k, t + 1)
        row = got[t]
        assert np.count_nonzero(row == -1) == k - keff
        valid = row[row >= 0]
        assert len(set(valid.tolist())) == keff          # unique
        assert valid.max() <= t                          # causal
        if t + 1 <= k:
            assert sorted(valid.tolist()) == list(range(t + 1))


def test_topk_ties_prefer_smaller_index_and_signed_zero_equal():
    sc = np.full((1, 8), 1.0, dtype=np.float32)
    sc[0, 2] = -0.0
    sc[0, 5] = 0.0
    sc[0, 6] = 0.0
    sc[0, 1] = 2.0
    sc = np.repeat(sc, 8, axis=0)
    cu_q = np.array([0, 1], dtype=np.int32)
    cu_k = np.array([0, 8], dtype=np.int32)
    got = oracle.topk(sc[:1], 7, rows=[0], cu_q=cu_q, cu_k=cu_k)   # pos = 7
    # 2.0 first, then the four 1.0s in index order (0,3,4,7), then zeros in index order (2,5)
    assert got[0].tolist() == [1, 0, 3, 4, 7, 2, 5]


# ------------------------------------------------------------------ sparse MLA pins

def test_sparse_mla_hand_worked_two_keys():
    g = _gold("mla_two_keys.json")
    q = np.zeros((2, 1, 2))
    q[:, 0, 0] = math.log(3.0)
    kv = np.array(g["kv"])
    idx = np.array(g["idx"], dtype=np.int32)
    o, lse = oracle.sparse_mla(q, kv, idx, g["scale"], d_v=g["Dv"])
    np.testing.assert_allclose(o, np.array(g["o"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=1e-15, atol=1e-15)


def _dense_causal_sdpa(q, kv, scale, d_v):
    """Textbook causal softmax attention with one shared K/V row per token (library SDPA)."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                 # [1,H,L,Dqk]
    kt = torch.from_numpy(kv)[None, None].expand(1, q.shape[1], -1, -1)
    vt = torch.from_numpy(kv[:, :d_v].copy())[None, None].expand(1, q.shape[1], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    # lse from numpy's own einsum loops (no BLAS): torch's first fp64 CPU einsum in a process
    # was seen to land 1e-9 away from later calls on the same inputs
    z = np.einsum("lhd,sd->hls", q, kv, optimize=False) * scale
    L = q.shape[0]
    z = np.where(np.tril(np.ones((L, L), dtype=bool))[None], z, -np.inf)
    m = z.max(axis=-1, keepdims=True)
    lse = (m[..., 0] + np.log(np.exp(z - m).sum(axis=-1)))
    return o[0].permute(1, 0, 2).numpy(), lse.T


def test_sparse_mla_equals_dense_causal_attention_when_k_covers_all():
    r = _rng(30)
    L, H, Dqk, Dv, k = 24, 4, 20, 12, 32
    q = r.standard_normal((L, H, Dqk))
    kv = r.standard_normal((L, Dqk))
    scale = 1.0 / math.sqrt(7.0)
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        idx[t, : t + 1] = r.permutation(t + 1)
    o, lse = oracle.sparse_mla(q, kv, idx, scale, d_v=Dv)
    o_ref, lse_ref = _dense_causal_sdpa(q, kv, scale, Dv)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_forward_with_k_at_least_L_is_dense_attention():
    # End to end: when index_topk >= L every causal key is selected, whatever the scores.
    r = _rng(31)
    L, HI, DI, H, Dqk, Dv = 16, 3, 8, 2, 12, 8
    o_sc, ix, o, lse = oracle.forward(r.standard_normal((L, HI, DI)), r.standard_normal((L, HI)),
                                      r.standard_normal((L, DI)), q := r.standard_normal((L, H, Dqk)),
                                      kv := r.standard_normal((L, Dqk)), topk_k=L, scale=0.3, d_v=Dv)
    o_ref, lse_ref = _dense_causal_sdpa(q, kv, 0.3, Dv)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_sparse_mla_permutation_invariant_and_masks_invalid_slots():
    r = _rng(32)
    L, H, Dqk, Dv, k = 30, 3, 16, 8, 10
    q = r.standard_normal((L, H, Dqk))
    kv = r.standard_normal((L, Dqk))
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        n = min(k, t + 1)
        idx[t, :n] = r.choice(t + 1, n, replace=False)
    o, lse = oracle.sparse_mla(q, kv, idx, 0.25, d_v=Dv)
    perm = np.stack([r.permutation(k) for _ in range(L)])
    idx_p = np.take_along_axis(idx, perm, axis=1)
    o2, lse2 = oracle.sparse_mla(q, kv, idx_p, 0.25, d_v=Dv)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12, atol=1e-13)
    # Slots that point past pos(t) (future keys) or past the sequence are ignored.
    idx_bad = idx.copy()
    for t in range(L - 1):
        free = np.where(idx_bad[t] == -1)[0]
        if len(free):
            idx_bad[t, free[0]] = t + 1 + (t % 3)
    o3, lse3 = oracle.sparse_mla(q, kv, idx_bad, 0.25, d_v=Dv)
    np.testing.assert_allclose(o3, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse3, lse, rtol=1e-12, atol=1e-13)


def test_sparse_mla_heads_share_the_latent_and_single_key_returns_value():
    r = _rng(33)
    L, H, Dqk, Dv, k = 9, 4, 10, 6, 4
    q = r.standard_normal((L, H, Dqk))
    q[:, 2] = q[:, 0]                                    # identical heads
    kv = r.standard_normal((L, Dqk))
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        n = min(k, t + 1)
        idx[t, :n] = np.arange(t + 1 - n, t + 1)
    o, lse = oracle.sparse_mla(q, kv, idx, 0.5, d_v=Dv)
    np.testing.assert_array_equal(o[:, 2], o[:, 0])
    np.testing.assert_array_equal(lse[:, 2], lse[:, 0])
    # a single valid key: o = value part of that latent row, lse = its logit
    one = np.full((L, k), -1, dtype=np.int32)
    one[:, 0] = 0
    o1, lse1 = oracle.sparse_mla(q, kv, one, 0.5, d_v=Dv)
    np.testing.assert_allclose(o1, np.broadcast_to(kv[0, :Dv], o1.shape), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse1, 0.5 * np.einsum("thd,d->th", q, kv[0]), rtol=1e-14, atol=1e-14)
    # no valid key at all: zeros and -inf
    none = np.full((L, k), -1, dtype=np.int32)
    o0, lse0 = oracle.sparse_mla(q, kv, none, 0.5, d_v=Dv)
    assert np.all(o0 == 0) and np.all(lse0 == -np.inf)


def test_decode_rows_equal_last_prefill_rows():
    # The ragged reading: a decode query at pos = len_k - 1 sees exactly what the last
    # prefill query of the same sequence sees.
    r = _rng(34)
    HI, DI, H, Dqk, Dv = 2, 8, 2, 12, 8
    lens = [13, 21, 5]
    k_all = r.standard_normal((sum(lens), DI))
    kv_all = r.standard_normal((sum(lens), Dqk))
    qI = r.standard_normal((3, HI, DI))
    w = r.standard_normal((3, HI))
    q = r.standard_normal((3, H, Dqk))
    cu_q = np.arange(4, dtype=np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    sc, ix, o, lse = oracle.forward(qI, w, k_all, q, kv_all, topk_k=6, scale=0.4, d_v=Dv, cu_q=cu_q, cu_k=cu_k)
    for b, Lb in enumerate(lens):
        s0 = cu_k[b]
        rows = [Lb - 1]
        qI_p = np.zeros((Lb, HI, DI)); qI_p[-1] = qI[b]
        w_p = np.zeros((Lb, HI)); w_p[-1] = w[b]
        q_p = np.zeros((Lb, H, Dqk)); q_p[-1] = q[b]
        sc_p, ix_p, o_p, lse_p = oracle.forward(qI_p[-1:], w_p[-1:], k_all[s0:s0 + Lb], q_p[-1:],
                                                kv_all[s0:s0 + Lb], topk_k=6, scale=0.4, d_v=Dv,
                                                rows=rows)
        np.testing.assert_array_equal(sc[b, :Lb], sc_p[0])
        np.testing.assert_array_equal(ix[b], ix_p[0])
        np.testing.assert_array_equal(o[b], o_p[0])


# ------------------------------------------------------------------ paged caches

def test_paged_layout_gives_the_packed_results_exactly():
    # Paged caches ("DeepSeek-V3.2" miles docs §5.3: KV cache pages of 64 tokens): reading the
    # keys through a shuffled block table must give bit for bit what the packed rows give, for
    # every oracle function (the same fp64 operations on the same values).
    import dsa_synth

    inp = dsa_synth.make_decode(4, 90, 400, topk=32, seed=41, q_per_seq=3)
    pg = dsa_synth.to_paged(inp, page_size=64, seed=5)
    assert int(pg["block_table"][0, 1]) != int(pg["block_table"][0, 0]) + 1 or \
        int(pg["block_table"][1, 0]) != int(pg["block_table"][0, -1]) + 1      # really shuffled
    kw = dict(cu_q=inp["cu_q"], cu_k=inp["cu_k"])
    T = inp["total_q"]
    sc = oracle.indexer(inp["q_idx"], inp["w"], inp["k_idx"], **kw)
    sc_p = oracle.indexer(inp["q_idx"], inp["w"], pg["k_idx"], block_table=pg["block_table"], **kw)
    np.testing.assert_array_equal(sc, sc_p)
    ix = oracle.topk(sc, 32, **kw)
    o, lse = oracle.sparse_mla(inp["q"], inp["kv"], ix, 0.3, **kw)
    o_p, lse_p = oracle.sparse_mla(inp["q"], pg["kv"], ix, 0.3, block_table=pg["block_table"], **kw)
    np.testing.assert_array_equal(o, o_p)
    np.testing.assert_array_equal(lse, lse_p)
    full = oracle.forward(inp["q_idx"], inp["w"], pg["k_idx"], inp["q"], pg["kv"], 32, 0.3,
                          block_table=pg["block_table"], **kw)
    np.testing.assert_array_equal(full[1], ix)
    # FP8 keys with per-token scales travel with their rows
    q8, qs = dsa_synth.quantize_e4m3_per_token(inp["q_idx"].float())
    k8, ks = dsa_synth.quantize_e4m3_per_token(inp["k_idx"].float())
    f8 = dict(inp, k_idx8=k8, k_scale=ks)
    pg8 = dsa_synth.to_paged(f8, page_size=64, seed=6)
    a = oracle.indexer_fp8(q8, qs, inp["w"], k8, ks, **kw)
    b = oracle.indexer_fp8(q8, qs, inp["w"], pg8["k_idx8"], pg8["k_scale"], block_table=pg8["block_table"], **kw)
    np.testing.assert_array_equal(a, b)
    # and the table really is consulted: a table pointing at the wrong pages changes the scores
    bad = pg["block_table"].clone()
    bad[0, 0], bad[0, 1] = bad[0, 1].clone(), bad[0, 0].clone()
    sc_bad = oracle.indexer(inp["q_idx"], inp["w"], pg["k_idx"], block_table=bad, **kw)
    assert not np.array_equal(sc_bad[:3], sc[:3])
    assert T == 12


# ------------------------------------------------- FP8 with ue8m0 block scales

def test_ue8m0_decoder_matches_library_cast():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    ours = np.array([oracle.ue8m0_value(i) for i in range(256)])
    assert np.isnan(ours[255]) and np.isnan(lib[255])
    np.testing.assert_array_equal(ours[:255], lib[:255])


def test_block_scaled_fp8_indexer_equals_float_indexer_on_dequantised_inputs():
    # 128-element blocks: one per (token, head) of q_I, one per token of k_I; scales 2^(e-127)
    import dsa_synth

    g = torch.Generator().manual_seed(61)
    T, H, D = 40, 5, 128
    q = torch.randn(T, H, D, generator=g) * torch.rand(T, H, 1, generator=g).mul(6).exp2()
    k = torch.randn(T, D, generator=g) * 3.0
    w = torch.randn(T, H, generator=g)
    q8, qe = dsa_synth.quantize_e4m3_ue8m0_blocks(q)
    k8, ke = dsa_synth.quantize_e4m3_ue8m0_blocks(k)
    assert qe.shape == (T, H) and ke.shape == (T,)
    got = oracle.indexer_fp8_block(q8, qe, w, k8, ke)
    lib_q = q8.view(torch.float8_e4m3fn).double() * qe.view(torch.float8_e8m0fnu).double()[:, :, None]
    lib_k = k8.view(torch.float8_e4m3fn).double() * ke.view(torch.float8_e8m0fnu).double()[:, None]
    ref = oracle.indexer(lib_q, w, lib_k)
    tri = np.tril(np.ones((T, T), dtype=bool))
    np.testing.assert_allclose(got[tri], ref[tri], rtol=1e-12, atol=1e-12)
    # each head's own scale: raising head 2's exponent by one doubles the score of a row that
    # weights only head 2 (positive homogeneity of ReLU), and leaves head 3's row unchanged
    w1 = torch.zeros(T, H)
    w1[:, 2] = 1.0
    qe2 = qe.clone()
    qe2[:, 2] += 1
    a = oracle.indexer_fp8_block(q8, qe, w1, k8, ke)
    b = oracle.indexer_fp8_block(q8, qe2, w1, k8, ke)
    np.testing.assert_array_equal(b[tri], 2.0 * a[tri])
    w3 = torch.zeros(T, H)
    w3[:, 3] = 1.0
    np.testing.assert_array_equal(oracle.indexer_fp8_block(q8, qe2, w3, k8, ke)[tri],
                                  oracle.indexer_fp8_block(q8, qe, w3, k8, ke)[tri])


# ------------------------------------------------------ key-cache write producer

def _cache_inputs(n, seed, positions):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(n, 128, generator=g, dtype=torch.float64) * 2 + 0.5
    kv = torch.randn(n, 576, generator=g, dtype=torch.float64)
    ln_w = torch.rand(128, generator=g, dtype=torch.float64) + 0.5
    ln_b = torch.randn(128, generator=g, dtype=torch.float64) * 0.1
    rms_w = torch.rand(512, generator=g, dtype=torch.float64) + 0.5
    inv_freq = torch.rand(32, generator=g, dtype=torch.float64) * 0.9 + 0.01
    pos = torch.tensor(positions, dtype=torch.int32)
    return k, kv, pos, ln_w, ln_b, rms_w, inv_freq


def test_cache_write_norms_match_library_at_position_zero():
    # position 0 rotates by nothing: the rows are torch's layer_norm / rms_norm
    eps = 1e-6
    k, kv, _, ln_w, ln_b, rms_w, inv_freq = _cache_inputs(6, 71, [0] * 6)
    ok, okv = oracle.cache_write(k, kv, torch.zeros(6, dtype=torch.int32), ln_w, ln_b, rms_w, inv_freq, eps)
    ref_k = torch.nn.functional.layer_norm(k, (128,), ln_w, ln_b, eps).numpy()
    ref_z = torch.nn.functional.rms_norm(kv[:, :512], (512,), rms_w, eps).numpy()
    np.testing.assert_allclose(ok, ref_k, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(okv[:, :512], ref_z, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(okv[:, 512:], kv[:, 512:].numpy())


def test_cache_write_rope_layouts_are_complex_rotations():
    # RoPE rotates pair i by pos * inv_freq[i] (multiplication by e^{i theta}); the indexer's
    # pairs are (i, i + 32) of its first 64 dims (non-interleaved), the latent's are
    # (512 + 2i, 513 + 2i) (interleaved)
    eps = 1e-6
    positions = [1, 7, 100, 4095, 65536, 163839]
    k, kv, pos, ln_w, ln_b, rms_w, inv_freq = _cache_inputs(len(positions), 72, positions)
    ok, okv = oracle.cache_write(k, kv, pos, ln_w, ln_b, rms_w, inv_freq, eps)
    theta = pos.double()[:, None] * inv_freq[None, :]
    rot = torch.polar(torch.ones_like(theta), theta)
    normed = torch.nn.functional.layer_norm(k, (128,), ln_w, ln_b, eps)
    zi = torch.complex(normed[:, :32], normed[:, 32:64]) * rot
    np.testing.assert_allclose(ok[:, :32], zi.real.numpy(), rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(ok[:, 32:64], zi.imag.numpy(), rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(ok[:, 64:], normed[:, 64:].numpy(), rtol=1e-12, atol=1e-12)
    zl = torch.view_as_complex(kv[:, 512:].reshape(-1, 32, 2).contiguous()) * rot
    np.testing.assert_allclose(okv[:, 512:], torch.view_as_real(zl).reshape(-1, 64).numpy(), rtol=1e-9, atol=1e-9)
    # the two layouts really differ: rotating the latent's dims non-interleaved would not match
    wrong = torch.complex(kv[:, 512:544], kv[:, 544:576]) * rot
    assert not np.allclose(okv[:, 512:544], wrong.real.numpy(), atol=1e-6)
