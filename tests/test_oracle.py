"""Pins of the CPU oracle against what the QUOKA write-up and plain
mathematics fix: hand-derived closed forms, invariants, special cases that
reduce to a library routine, and brute force on tiny inputs.

Each pin is chosen so that a plausible slip in the oracle (a dropped minus
sign, a mean over the wrong axis, a transposed operand, min for max, a wrong
head-to-group map, a wrong causal direction) fails at least one test here.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import quoka_oracle as orc
from sparse_kv_selection_quoka_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- step (a)

def test_query_scores_hand_worked(golden):
    g = golden["query_scores"]
    SQ = orc.query_scores(np.array(g["Q"], dtype=np.float64))
    np.testing.assert_allclose(SQ, np.array(g["SQ"]), rtol=0, atol=1e-15)


def test_query_scores_range_and_scale_invariance():
    Q = rng(1).standard_normal((2, 3, 17, 8))
    SQ = orc.query_scores(Q)
    assert np.all(SQ >= -1 - 1e-12) and np.all(SQ <= 1 + 1e-12)
    # rescaling one whole head by c > 0 rescales its mean by c: SQ unchanged
    Q2 = Q.copy()
    Q2[1, 2] *= 7.5
    Q2[0, 0] *= 0.01
    np.testing.assert_allclose(orc.query_scores(Q2), SQ, atol=1e-12)
    # rescaling a single token changes the mean, so SQ must change somewhere
    Q3 = Q.copy()
    Q3[0, 1, 4] *= 5.0
    assert np.abs(orc.query_scores(Q3)[0, 1] - SQ[0, 1]).max() > 1e-3


def test_query_scores_single_token_is_minus_one():
    # with one token the mean is that token: cos = 1, SQ = -1
    Q = rng(2).standard_normal((1, 4, 1, 16))
    np.testing.assert_allclose(orc.query_scores(Q), -1.0, atol=1e-14)


def test_query_scores_per_head_mean():
    # two heads holding the same tokens in different order give the same
    # per-token scores (the mean is over tokens, not over heads)
    base = rng(3).standard_normal((9, 5))
    perm = rng(4).permutation(9)
    Q = np.stack([base, base[perm], 3.0 * base + 1.0])[None]
    SQ = orc.query_scores(Q)
    np.testing.assert_allclose(SQ[0, 1], SQ[0, 0][perm], atol=1e-14)
    # a head with a different mean gives different scores
    assert np.abs(SQ[0, 2] - SQ[0, 0]).max() > 1e-3


# ----------------------------------------------------------------- step (b)

def _rank_by_counting(v):
    """Brute force: the rank of entry t is the number of entries that beat it
    (a larger value, or an equal value at a lower position)."""
    n = len(v)
    rank = np.zeros(n, dtype=np.int64)
    for t in range(n):
        for u in range(n):
            if v[u] > v[t] or (v[u] == v[t] and u < t):
                rank[t] += 1
    return rank


def test_select_queries_hand_worked(golden):
    g = golden["query_scores"]
    q_idx = orc.select_queries(np.array(g["SQ"]), g["NQ"])
    assert q_idx.tolist() == g["q_idx"]


@pytest.mark.parametrize("seed", range(6))
def test_select_queries_brute_force(seed):
    r = rng(100 + seed)
    L = int(r.integers(1, 20))
    NQ = int(r.integers(1, L + 1))
    # coarse values force ties
    SQ = np.round(r.uniform(-1, 1, size=(2, 3, L)), 1)
    q_idx = orc.select_queries(SQ, NQ)
    for b in range(2):
        for h in range(3):
            rank = _rank_by_counting(SQ[b, h])
            expect = [int(np.where(rank == k)[0][0]) for k in range(NQ)]
            assert q_idx[b, h].tolist() == expect


def test_select_queries_rejects_bad_nq():
    with pytest.raises(ValueError):
        orc.select_queries(np.zeros((1, 1, 4)), 5)
    with pytest.raises(ValueError):
        orc.select_queries(np.zeros((1, 1, 4)), 0)


# ----------------------------------------------------------------- step (c)

def test_group_queries_hand_worked(golden):
    g = golden["group_queries"]
    Qg = orc.group_queries(np.array(g["Q"], dtype=np.float64),
                           np.array(g["q_idx"]), g["nkv"])
    np.testing.assert_allclose(Qg, np.array(g["Q_group"]), atol=1e-15)


def test_group_queries_g1_is_normalised_choice():
    Q = rng(5).standard_normal((2, 3, 11, 8))
    q_idx = orc.select_queries(orc.query_scores(Q), 4)
    Qg = orc.group_queries(Q, q_idx, nkv=3)          # G = 1
    chosen = np.take_along_axis(Q, q_idx[..., None], axis=2)
    np.testing.assert_allclose(Qg, chosen / np.linalg.norm(chosen, axis=-1, keepdims=True),
                               atol=1e-14)


def test_group_queries_identical_heads_and_norm_bound():
    r = rng(6)
    one = r.standard_normal((1, 1, 10, 6))
    Q = np.repeat(one, 4, axis=1)                     # 4 identical heads, G = 4
    q_idx = orc.select_queries(orc.query_scores(Q), 3)
    Qg = orc.group_queries(Q, q_idx, nkv=1)
    chosen = one[0, 0, q_idx[0, 0]]
    np.testing.assert_allclose(Qg[0, 0], chosen / np.linalg.norm(chosen, axis=-1, keepdims=True),
                               atol=1e-14)
    # a mean of unit vectors has norm <= 1
    Q = r.standard_normal((2, 8, 12, 6))
    Qg = orc.group_queries(Q, orc.select_queries(orc.query_scores(Q), 5), nkv=2)
    assert np.all(np.linalg.norm(Qg, axis=-1) <= 1 + 1e-12)


def test_group_queries_head_to_group_map():
    # nq = 4, nkv = 2: heads 0,1 -> KV head 0; heads 2,3 -> KV head 1
    Q = np.zeros((1, 4, 2, 2))
    Q[0, 0, :] = [1, 0]
    Q[0, 1, :] = [1, 0]
    Q[0, 2, :] = [0, 1]
    Q[0, 3, :] = [0, 1]
    q_idx = np.zeros((1, 4, 1), dtype=np.int64)
    Qg = orc.group_queries(Q, q_idx, nkv=2)
    np.testing.assert_allclose(Qg[0, 0, 0], [1, 0])
    np.testing.assert_allclose(Qg[0, 1, 0], [0, 1])


# ----------------------------------------------------------------- step (d)

def test_key_scores_hand_worked(golden):
    g = golden["key_scores"]
    S = orc.key_scores(np.array(g["Q_group"], dtype=np.float64), np.array(g["K"], dtype=np.float64))
    np.testing.assert_allclose(S, np.array(g["S_agg"]), atol=1e-15)
    assert orc.select_keys(S, g["BSA"]).tolist() == g["sel"]


def test_key_scores_range_and_key_scale_invariance():
    r = rng(7)
    Q = r.standard_normal((1, 6, 20, 8))
    K = r.standard_normal((1, 2, 33, 8))
    res = orc.select(Q, K, NQ=5, BSA=10)
    S = res["S_agg"]
    assert np.all(S >= -1 - 1e-12) and np.all(S <= 1 + 1e-12)
    K2 = K * r.uniform(0.1, 10.0, size=(1, 2, 33, 1))
    np.testing.assert_allclose(orc.key_scores(res["Q_group"], K2), S, atol=1e-13)


def test_key_scores_equal_mean_of_per_head_cosines():
    """The page's prose describes the aggregation as an average over the
    group's heads of the per-query cosine scores, then a max over the chosen
    queries; its code normalises, averages the queries and multiplies. By
    linearity the two agree; this recomputes the prose version with explicit
    per-pair cosines."""
    r = rng(8)
    b, nq, nkv, L, T, d, NQ = 2, 6, 2, 9, 15, 5, 4
    G = nq // nkv
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    res = orc.select(Q, K, NQ=NQ, BSA=3)
    q_idx = res["q_idx"]
    for bi in range(b):
        for j in range(nkv):
            for tau in range(T):
                k = K[bi, j, tau]
                best = -math.inf
                for i in range(NQ):
                    cs = []
                    for g in range(G):
                        q = Q[bi, j * G + g, q_idx[bi, j * G + g, i]]
                        cs.append(float(q @ k) / (np.linalg.norm(q) * np.linalg.norm(k)))
                    best = max(best, sum(cs) / G)
                assert abs(res["S_agg"][bi, j, tau] - best) < 1e-13


def test_key_scores_query_scale_invariance_within_choice():
    # rescaling a chosen query leaves S unchanged when the choice is held fixed
    r = rng(9)
    Q = r.standard_normal((1, 4, 10, 6))
    K = r.standard_normal((1, 2, 12, 6))
    res = orc.select(Q, K, NQ=3, BSA=4)
    Q2 = Q.copy()
    Q2[0, 1, res["q_idx"][0, 1, 0]] *= 4.0
    res2 = orc.select(Q2, K, NQ=3, BSA=4, override_q_idx=res["q_idx"])
    np.testing.assert_allclose(res2["S_agg"], res["S_agg"], atol=1e-13)


# ----------------------------------------------------------------- step (e)

def test_select_keys_ties(golden):
    g = golden["select_keys_ties"]
    S = np.array(g["S_agg"])
    for bsa, expect in g["cases"]:
        assert orc.select_keys(S, bsa)[0, 0].tolist() == expect


@pytest.mark.parametrize("seed", range(5))
def test_select_keys_exhaustive(seed):
    """On tiny inputs with distinct scores, the selected set is the size-BSA
    subset with the largest score sum, found by enumerating all subsets."""
    r = rng(200 + seed)
    T = int(r.integers(1, 13))
    S = r.permutation(T).astype(np.float64)[None, None] + r.uniform(0, 0.5)
    S = S * r.choice([-1.0, 1.0])
    for bsa in range(0, min(T, 5) + 1):
        best = max(itertools.combinations(range(T), bsa),
                   key=lambda c: sum(S[0, 0, list(c)]) if c else 0.0)
        assert orc.select_keys(S, bsa)[0, 0].tolist() == sorted(best)


def test_select_keys_separation_and_edges():
    r = rng(10)
    S = np.round(r.uniform(-1, 1, size=(2, 3, 57)), 2)
    sel = orc.select_keys(S, 20)
    for b in range(2):
        for j in range(3):
            s = set(sel[b, j].tolist())
            assert sel[b, j].tolist() == sorted(s) and len(s) == 20
            inside = S[b, j, sorted(s)]
            outside = S[b, j, [t for t in range(57) if t not in s]]
            assert inside.min() >= outside.max()
            # among equal scores at the boundary the lower indices are taken
            thr = inside.min()
            eq_in = [t for t in s if S[b, j, t] == thr]
            eq_out = [t for t in range(57) if t not in s and S[b, j, t] == thr]
            if eq_in and eq_out:
                assert max(eq_in) < min(eq_out)
    assert orc.select_keys(np.zeros((1, 2, 0)), 5).shape == (1, 2, 0)
    assert orc.select_keys(S, 100).shape == (2, 3, 57)


# ------------------------------------------------------------- steps (f)(g)

def _sdpa_dense_reference(Q, K, V, Kc, Vc, scale):
    """Dense attention over [prior keys ; chunk keys] with the chunk causal,
    through torch's library scaled_dot_product_attention in float64."""
    b, nq, L, d = Q.shape
    nkv = Kc.shape[1]
    G = nq // nkv
    keys = torch.from_numpy(np.concatenate([K, Kc], axis=2)).double()
    vals = torch.from_numpy(np.concatenate([V, Vc], axis=2)).double()
    keys = keys.repeat_interleave(G, dim=1)
    vals = vals.repeat_interleave(G, dim=1)
    T = K.shape[2]
    mask = torch.ones(L, T + L, dtype=torch.bool)
    mask[:, T:] = torch.tril(torch.ones(L, L, dtype=torch.bool))
    q = torch.from_numpy(np.ascontiguousarray(Q)).double()
    O = torch.nn.functional.scaled_dot_product_attention(q, keys, vals, attn_mask=mask, scale=scale)
    logits = (q @ keys.transpose(-1, -2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
    return O.numpy(), lse.numpy()


@pytest.mark.parametrize("shape", [(1, 4, 2, 8, 13, 6), (2, 6, 3, 16, 0, 5), (1, 3, 1, 4, 9, 7)])
def test_dense_reduction_equals_sdpa(shape):
    """NQ = BCP and BSA = T select everything: the step is dense causal
    attention over prior + chunk keys."""
    b, nq, nkv, d, T, L = shape
    r = rng(11)
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    V = r.standard_normal((b, nkv, T, d))
    Kc = r.standard_normal((b, nkv, L, d))
    Vc = r.standard_normal((b, nkv, L, d))
    res = orc.prefill_chunk(Q, K, V, Kc, Vc, NQ=L, BSA=T)
    assert res["sel"].shape == (b, nkv, T)
    O_ref, lse_ref = _sdpa_dense_reference(Q, K, V, Kc, Vc, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(res["O"], O_ref, atol=1e-12)
    np.testing.assert_allclose(res["LSE"], lse_ref, atol=1e-12)


def test_attention_first_query_without_prior_is_value(golden):
    r = rng(12)
    Q = r.standard_normal((1, 4, 6, 8))
    Kc = r.standard_normal((1, 2, 6, 8))
    Vc = r.standard_normal((1, 2, 6, 8))
    empty = np.zeros((1, 2, 0, 8))
    O, _ = orc.sparse_attention(Q, empty, empty, np.zeros((1, 2, 0), dtype=np.int64), Kc, Vc)
    for h in range(4):
        np.testing.assert_allclose(O[0, h, 0], Vc[0, h // 2, 0], atol=1e-15)


def test_attention_identical_keys_is_mean_of_visible_values():
    r = rng(13)
    T, L, d = 7, 5, 4
    krow = r.standard_normal(d)
    K = np.broadcast_to(krow, (1, 1, T, d)).copy()
    Kc = np.broadcast_to(krow, (1, 1, L, d)).copy()
    V = r.standard_normal((1, 1, T, d))
    Vc = r.standard_normal((1, 1, L, d))
    Q = r.standard_normal((1, 2, L, d))
    sel = np.array([[[1, 4, 6]]])
    O, _ = orc.sparse_attention(Q, K, V, sel, Kc, Vc)
    for t in range(L):
        visible = np.concatenate([V[0, 0, [1, 4, 6]], Vc[0, 0, :t + 1]])
        for h in range(2):
            np.testing.assert_allclose(O[0, h, t], visible.mean(axis=0), atol=1e-14)


def test_attention_head_map_and_selected_set_order():
    r = rng(14)
    b, nq, nkv, T, L, d = 1, 4, 2, 10, 3, 4
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    Kc = r.standard_normal((b, nkv, L, d))
    V = np.empty((b, nkv, T, d))
    Vc = np.empty((b, nkv, L, d))
    V[:, 0] = -3.0
    Vc[:, 0] = -3.0
    V[:, 1] = 7.0
    Vc[:, 1] = 7.0
    sel = np.array([[[0, 2, 5], [1, 8, 9]]])
    O, lse = orc.sparse_attention(Q, K, V, sel, Kc, Vc)
    np.testing.assert_allclose(O[0, :2], -3.0, atol=1e-13)
    np.testing.assert_allclose(O[0, 2:], 7.0, atol=1e-13)
    # attention is a set function of the selected keys
    V = r.standard_normal((b, nkv, T, d))
    Vc = r.standard_normal((b, nkv, L, d))
    O1, l1 = orc.sparse_attention(Q, K, V, sel, Kc, Vc)
    O2, l2 = orc.sparse_attention(Q, K, V, sel[:, :, ::-1].copy(), Kc, Vc)
    np.testing.assert_allclose(O1, O2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)


def test_attention_lse_merges_two_key_sets():
    """LSE is the log partition function: attention over selected set A and
    over set B (each with the chunk keys) merge into attention over A u B
    once the shared chunk-key part is counted once. Check via T = 0 chunk-only
    attention: Z(A u chunk) = Z(A only) + Z(chunk only)."""
    r = rng(15)
    b, nq, nkv, T, L, d = 1, 2, 1, 9, 4, 6
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    V = r.standard_normal((b, nkv, T, d))
    Kc = r.standard_normal((b, nkv, L, d))
    Vc = r.standard_normal((b, nkv, L, d))
    sel = np.array([[[0, 3, 4, 8]]])
    O, lse = orc.sparse_attention(Q, K, V, sel, Kc, Vc)
    # chunk-only attention
    e = np.zeros((b, nkv, 0, d))
    Oc, lc = orc.sparse_attention(Q, e, e, np.zeros((b, nkv, 0), dtype=np.int64), Kc, Vc)
    # selected-only part computed by the torch library routine
    scale = 1.0 / math.sqrt(d)
    q = torch.from_numpy(Q).double()
    ks = torch.from_numpy(K[:, :, sel[0, 0]]).double().repeat_interleave(nq, dim=1)
    vs = torch.from_numpy(V[:, :, sel[0, 0]]).double().repeat_interleave(nq, dim=1)
    Os = torch.nn.functional.scaled_dot_product_attention(q, ks, vs, scale=scale).numpy()
    ls = torch.logsumexp(q @ ks.transpose(-1, -2) * scale, dim=-1).numpy()
    Z = np.exp(ls) + np.exp(lc)
    np.testing.assert_allclose(lse, np.log(Z), atol=1e-12)
    merged = (np.exp(ls)[..., None] * Os + np.exp(lc)[..., None] * Oc) / Z[..., None]
    np.testing.assert_allclose(O, merged, atol=1e-12)


# ------------------------------------------------------------- whole step

def test_planted_heavy_keys_are_selected_llama_shape():
    """Sanity (not parity): on the Llama-3.2-3B-shaped synthetic layer the
    chosen queries are the planted outliers, and the planted heavy keys land
    in the 25% key budget far more often than chance (25%). The rank-paired
    group mean mixes outlier directions across heads, so not every heavy key
    is kept; a sign slip or a min-for-max would drop the rate to chance or
    below."""
    x = inputs.make_workload(1)
    res = orc.select(x.Q, x.K, x.NQ, x.BSA)
    out_pos = x.meta["outlier_pos"]
    G = x.Q.shape[1] // x.K.shape[1]
    for h in range(x.Q.shape[1]):
        assert set(res["q_idx"][0, h].tolist()) <= set(out_pos[0, h // G].tolist())
    for j in range(x.K.shape[1]):
        kept = np.isin(x.meta["heavy_pos"][0, j], res["sel"][0, j]).mean()
        assert kept >= 0.75


def test_attention_rows_match_sdpa_dense():
    """The row-by-row attention used on large workloads, pinned to torch's
    library attention in the dense reduction (everything selected)."""
    r = rng(16)
    b, nq, nkv, d, T, L = 2, 4, 2, 8, 11, 6
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    V = r.standard_normal((b, nkv, T, d))
    Kc = r.standard_normal((b, nkv, L, d))
    Vc = r.standard_normal((b, nkv, L, d))
    sel = np.broadcast_to(np.arange(T), (b, nkv, T))
    O_ref, lse_ref = _sdpa_dense_reference(Q, K, V, Kc, Vc, 1.0 / math.sqrt(d))
    rows = [(bi, h, t) for bi in range(b) for h in range(nq) for t in range(L)]
    O_rows, lse_rows = orc.sparse_attention_rows(Q, K, V, sel, Kc, Vc, rows)
    for n, (bi, h, t) in enumerate(rows):
        np.testing.assert_allclose(O_rows[n], O_ref[bi, h, t], atol=1e-12)
        assert abs(lse_rows[n] - lse_ref[bi, h, t]) < 1e-12


# ------------------------------------------------ dot-product score variant
# [QUOKA §2.2] compares its cosine score with the standard dot-product score;
# the oracle's dot_product=True drops the L2 normalisation of the chosen
# queries and of the keys and keeps everything else.

def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_dot_product_equals_cosine_on_unit_vectors():
    """With every query and key of unit norm the two scores coincide, so
    the whole selection does too."""
    r = rng(21)
    Q = _unit_rows(r.standard_normal((2, 6, 12, 8)))
    K = _unit_rows(r.standard_normal((2, 3, 40, 8)))
    cos = orc.select(Q, K, NQ=4, BSA=9)
    dot = orc.select(Q, K, NQ=4, BSA=9, dot_product=True)
    np.testing.assert_array_equal(dot["q_idx"], cos["q_idx"])
    np.testing.assert_allclose(dot["S_agg"], cos["S_agg"], atol=1e-14)
    np.testing.assert_array_equal(dot["sel"], cos["sel"])


def test_dot_product_scales_with_the_keys_and_not_with_their_norm():
    """Scaling all keys by c > 0 scales the dot-product score by c and keeps
    the selection; scaling one key changes its score by that factor only
    (the cosine score ignores both)."""
    r = rng(22)
    Q = r.standard_normal((1, 4, 10, 6))
    K = r.standard_normal((1, 2, 25, 6))
    base = orc.select(Q, K, NQ=3, BSA=7, dot_product=True)
    scaled = orc.select(Q, 3.5 * K, NQ=3, BSA=7, dot_product=True)
    np.testing.assert_allclose(scaled["S_agg"], 3.5 * base["S_agg"], rtol=1e-13)
    np.testing.assert_array_equal(scaled["sel"], base["sel"])
    K2 = K.copy()
    K2[0, 1, 5] *= 0.25
    one = orc.select(Q, K2, NQ=3, BSA=7, dot_product=True)
    expect = base["S_agg"].copy()
    expect[0, 1, 5] = 0.25 * base["S_agg"][0, 1, 5]
    np.testing.assert_allclose(one["S_agg"], expect, rtol=1e-13, atol=1e-15)
    cos1 = orc.select(Q, K, NQ=3, BSA=7)
    cos2 = orc.select(Q, K2, NQ=3, BSA=7)
    np.testing.assert_allclose(cos2["S_agg"], cos1["S_agg"], atol=1e-13)


def test_dot_product_is_mean_of_per_head_raw_dots():
    """By linearity, the max over chosen queries of (mean of the group's raw
    chosen queries) . k equals the max of the mean of the per-head raw dot
    products, computed here pair by pair with numpy.einsum."""
    r = rng(23)
    b, nq, nkv, L, T, d, NQ = 2, 6, 2, 9, 15, 5, 4
    G = nq // nkv
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    res = orc.select(Q, K, NQ=NQ, BSA=3, dot_product=True)
    q_idx = res["q_idx"]
    chosen = np.take_along_axis(Q, q_idx[..., None], axis=2)          # (b, nq, NQ, d)
    per_head = np.einsum("bhid,bhtd->bhit", chosen, np.repeat(K, G, axis=1))
    expect = per_head.reshape(b, nkv, G, NQ, T).mean(axis=2).max(axis=2)
    np.testing.assert_allclose(res["S_agg"], expect, atol=1e-12)
    # and the query choice is the cosine variant's (steps (a), (b) unchanged)
    np.testing.assert_array_equal(q_idx, orc.select(Q, K, NQ=NQ, BSA=3)["q_idx"])


# ------------------------------------------- prior keys split over ranks
# The sharded step (sparse_kv_selection_quoka_b200.sharded) rests on two
# facts pinned here on the oracle: the union of every shard's top-BSA holds
# the global top-BSA, and softmax partials over disjoint key sets merge by
# their log-sum-exp.

def test_attention_without_chunk_keys():
    """include_chunk=False over every prior key is dense non-causal attention
    over K (torch's library attention); with no selected key the rows are
    empty (O = 0, LSE = -inf)."""
    r = rng(31)
    b, nq, nkv, d, T, L = 1, 4, 2, 8, 9, 5
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    V = r.standard_normal((b, nkv, T, d))
    Kc = r.standard_normal((b, nkv, L, d))
    Vc = r.standard_normal((b, nkv, L, d))
    sel = np.broadcast_to(np.arange(T), (b, nkv, T))
    O, lse = orc.sparse_attention(Q, K, V, sel, Kc, Vc, include_chunk=False)
    G = nq // nkv
    Kr = torch.from_numpy(np.repeat(K, G, axis=1))
    Vr = torch.from_numpy(np.repeat(V, G, axis=1))
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(Q), Kr, Vr).numpy()
    np.testing.assert_allclose(O, ref, atol=1e-12)
    O0, lse0 = orc.sparse_attention(Q, K, V, np.zeros((b, nkv, 0), dtype=np.int64), Kc, Vc,
                                    include_chunk=False)
    assert np.all(O0 == 0.0) and np.all(np.isneginf(lse0))


def _merge_shard_selection(S_agg, T_shards, BSA):
    """Global top-BSA from the shards' own top-BSA candidates, ranked over
    their concatenation (shard order, ascending positions) with ties to the
    earlier entry."""
    offs = np.cumsum([0] + list(T_shards))
    b, nkv, _ = S_agg.shape
    n = min(BSA, offs[-1])
    out = np.empty((b, nkv, n), dtype=np.int64)
    for bi in range(b):
        for j in range(nkv):
            cand = []
            for r, Tr in enumerate(T_shards):
                local = orc.select_keys(S_agg[bi:bi + 1, j:j + 1, offs[r]:offs[r + 1]], BSA)[0, 0]
                cand.extend(int(offs[r] + t) for t in local)
            cand = np.array(cand, dtype=np.int64)
            sc = S_agg[bi, j, cand]
            order = np.lexsort((np.arange(len(cand)), -sc))
            out[bi, j] = np.sort(cand[order[:n]])
    return out


@pytest.mark.parametrize("T_shards", [(40, 40), (30, 11, 0, 25), (5, 70)])
def test_shard_candidates_hold_the_global_selection(T_shards):
    """Merging the shards' top-BSA gives exactly the one-device top-BSA,
    ties included (scores drawn on a coarse grid, so many tie)."""
    r = rng(32)
    T = sum(T_shards)
    S = np.round(r.standard_normal((2, 3, T)) * 4) / 4     # many exact ties
    for BSA in (1, 7, 20, T):
        np.testing.assert_array_equal(_merge_shard_selection(S, T_shards, BSA), orc.select_keys(S, BSA))


def test_lse_merge_of_shard_partials_is_the_whole_attention():
    """The softmax over a key set split into shards (chunk keys on the first
    one only) is the log-sum-exp merge of the per-shard softmaxes."""
    r = rng(33)
    b, nq, nkv, d, L = 1, 4, 2, 8, 6
    T_shards = (7, 0, 5)
    T = sum(T_shards)
    offs = np.cumsum([0] + list(T_shards))
    Q = r.standard_normal((b, nq, L, d))
    K = r.standard_normal((b, nkv, T, d))
    V = r.standard_normal((b, nkv, T, d))
    Kc = r.standard_normal((b, nkv, L, d))
    Vc = r.standard_normal((b, nkv, L, d))
    sel = np.sort(r.permutation(T)[:8])
    full, full_lse = orc.sparse_attention(Q, K, V, np.broadcast_to(sel, (b, nkv, 8)), Kc, Vc)
    Os, ls = [], []
    for rk in range(len(T_shards)):
        mine = sel[(sel >= offs[rk]) & (sel < offs[rk + 1])] - offs[rk]
        Ks, Vs = K[:, :, offs[rk]:offs[rk + 1]], V[:, :, offs[rk]:offs[rk + 1]]
        O_r, l_r = orc.sparse_attention(Q, Ks, Vs, np.broadcast_to(mine, (b, nkv, len(mine))), Kc, Vc,
                                        include_chunk=(rk == 0))
        Os.append(O_r)
        ls.append(l_r)
    lse = np.logaddexp.reduce(np.stack(ls), axis=0)
    w = np.exp(np.stack(ls) - lse)
    O = (w[..., None] * np.stack(Os)).sum(axis=0)
    np.testing.assert_allclose(O, full, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, atol=1e-12)
