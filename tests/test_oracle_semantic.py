"""Pins of the oracle's semantic-block index ("Coarse Semantic Blocks ...", Abstract):
Lloyd's k-means over the prompt's keys, centroid scoring, cluster selection and attention
over the selected clusters' members plus the tokens after the prompt.

The clustering definition itself is a reading (parity unpinned); these tests pin its
implementation by properties that hold for Lloyd's algorithm, and the scoring and
attention by special cases that reduce to known results:
- the k-means objective never increases from one iteration to the next;
- a converged partition is a fixed point (nearest centroid, centroid = member mean);
- keys placed exactly at C separated points are recovered after one iteration;
- one token per cluster reduces to token-level scoring and selection;
- a cluster's score is the mean of its members' exact scores;
- a budget covering every cluster is dense attention;
- a planted non-contiguous cluster is selected.
"""
import math

import numpy as np

from oracle import formats as F
from oracle import method as M
from oracle import step as ST


def _bf(x):
    return F.f32_to_bf16_rne(np.asarray(x, dtype=np.float32))


def _mixture(rng, L, d, m, spread=4.0, noise=0.5):
    centres = rng.standard_normal((m, d)) * spread
    lab = rng.integers(0, m, size=L)
    return _bf(centres[lab] + noise * rng.standard_normal((L, d)))


def test_objective_never_increases():
    rng = np.random.default_rng(1)
    k = _mixture(rng, 600, 32, 10)
    prev = math.inf
    for it in range(1, 9):
        a, c = M.kmeans_keys(k, 12, it)
        obj = M.kmeans_objective(k, a, c)
        assert obj <= prev * (1 + 1e-12), (it, obj, prev)
        prev = obj


def test_converged_partition_is_a_fixed_point():
    rng = np.random.default_rng(2)
    k = _mixture(rng, 400, 16, 6, spread=6.0, noise=0.3)
    a30, c30 = M.kmeans_keys(k, 6, 30)
    a31, c31 = M.kmeans_keys(k, 6, 31)
    assert np.array_equal(a30, a31)
    x = F.bf16_to_f64(k)
    for t in range(len(x)):                       # nearest centroid, by a loop per point
        dist = [math.fsum((x[t] - c30[j]) ** 2) for j in range(6)]
        assert a30[t] == int(np.argmin(dist))
    for j in range(6):                            # centroid = member mean
        mem = x[a30 == j]
        if len(mem):
            want = [math.fsum(mem[:, i]) / len(mem) for i in range(x.shape[1])]
            assert np.allclose(c30[j], want, rtol=0, atol=1e-12)


def test_exactly_placed_keys_are_recovered_in_one_iteration():
    rng = np.random.default_rng(3)
    C, L0, d = 5, 200, 8
    points = np.zeros((C, d))
    points[np.arange(C), np.arange(C)] = 8.0      # separated, exact in BF16
    lab = rng.integers(0, C, size=L0)
    lab[(np.arange(C) * L0) // C] = np.arange(C)   # the seeds hold one point each
    k = _bf(points[lab])
    a, c = M.kmeans_keys(k, C, 1)
    assert np.array_equal(a, lab)
    assert np.array_equal(c, points)


def test_one_token_per_cluster_is_token_level():
    rng = np.random.default_rng(4)
    L0, d, G, B = 300, 16, 4, 20
    k = _bf(rng.standard_normal((L0, d)))
    q = _bf(rng.standard_normal((G, d)))
    a, c = M.kmeans_keys(k, L0, 3)                # S = 1: every key seeds its own cluster
    assert np.array_equal(a, np.arange(L0))
    x, qbar = F.bf16_to_f64(k), F.bf16_to_f64(q).mean(axis=0)
    exact = np.array([math.fsum(x[t] * qbar) for t in range(L0)])
    beta = M.semantic_block_scores(q, c)
    assert np.allclose(beta, exact, rtol=0, atol=1e-12)
    order = sorted(range(L0), key=lambda t: (-exact[t], t))[:B]
    assert M.select_blocks(beta, B, np.zeros(0, dtype=np.int64)).tolist() == sorted(order)


def test_cluster_score_is_the_mean_member_score():
    rng = np.random.default_rng(5)
    k = _mixture(rng, 500, 32, 7)
    q = _bf(rng.standard_normal((3, 32)))
    a, c = M.kmeans_keys(k, 9, 5)
    x, qbar = F.bf16_to_f64(k), F.bf16_to_f64(q).mean(axis=0)
    beta = M.semantic_block_scores(q, c)
    for j in range(9):
        mem = np.nonzero(a == j)[0]
        if len(mem):
            want = math.fsum(math.fsum(x[t] * qbar) for t in mem) / len(mem)
            assert abs(beta[j] - want) <= 1e-10 * max(1.0, abs(want))


def test_budget_covering_every_cluster_is_dense_attention():
    rng = np.random.default_rng(6)
    L0, L, d, G = 250, 260, 16, 2
    k = _mixture(rng, L, d, 4)
    v = _bf(rng.standard_normal((L, d)))
    q = _bf(rng.standard_normal((G, d)))
    p = ST.SemanticParams(S=32, budget=8, iters=4, scale=0.25, v_dtype="bf16")
    r = ST.decode_row_semantic(p, k, v, q, L0, L)
    assert r["tokens"].tolist() == list(range(L))
    x, vv, qq = F.bf16_to_f64(k), F.bf16_to_f64(v), F.bf16_to_f64(q)
    for h in range(G):
        logits = [0.25 * math.fsum(qq[h] * x[t]) for t in range(L)]
        m = max(logits)
        w = [math.exp(z - m) for z in logits]
        z = math.fsum(w)
        want = [math.fsum(w[t] * vv[t, i] for t in range(L)) / z for i in range(d)]
        assert np.allclose(r["out"][h], want, rtol=1e-12, atol=1e-12)


def test_planted_non_contiguous_cluster_is_selected():
    rng = np.random.default_rng(7)
    L0, L, d, G = 1000, 1010, 32, 4
    x = rng.standard_normal((L, d))
    m = np.zeros(d)
    m[0] = 1.0
    planted = np.sort(rng.choice(L0, size=40, replace=False))      # scattered positions
    x[planted] = 6.0 * m + 0.2 * rng.standard_normal((40, d))
    k = _bf(x)
    v = _bf(rng.standard_normal((L, d)))
    q = _bf(2.0 * m[None, :] + 0.1 * rng.standard_normal((G, d)))
    p = ST.SemanticParams(S=50, budget=1, iters=8, scale=1 / math.sqrt(d), v_dtype="bf16")
    r = ST.decode_row_semantic(p, k, v, q, L0, L)
    members = np.nonzero(r["assign"] == r["sel"][0])[0]
    assert set(planted.tolist()) <= set(members.tolist())
    assert set(range(L0, L)) <= set(r["tokens"].tolist())
    assert np.all(np.diff(r["tokens"]) > 0)


# ---- the float32 definition a kernel matches bit for bit --------------------------------------

def test_f32_distance_is_summed_in_float32_in_dimension_order():
    """Key (4096, 1, 1) against seeds (0, 0, 0) and (0, 1, 0): squared terms 2^24, 1, 1.
    In float32, in dimension order, both distances are 2^24, a tie won by cluster 0. In
    float64 (2^24 + 2 against 2^24 + 1), or in float32 in reversed order (2^24 + 2 against
    2^24), cluster 1 wins."""
    k = _bf(np.array([[0.0, 0.0, 0.0], [0.0, 1.0, 0.0], [4096.0, 1.0, 1.0]]))
    a32, _ = M.kmeans_keys_f32(k, 2, 1)
    a64, _ = M.kmeans_keys(k, 2, 1)
    assert a32.tolist() == [0, 1, 0]
    assert a64.tolist() == [0, 1, 1]


def test_f32_centroid_sums_members_in_token_order():
    """One cluster of 2^24, 1, -2^24: in float32 in token order the 1 is lost (mean 0);
    the exact mean is 1/3."""
    k = _bf(np.array([[2.0 ** 24], [1.0], [-(2.0 ** 24)]]))
    _, c32 = M.kmeans_keys_f32(k, 1, 1)
    _, c64 = M.kmeans_keys(k, 1, 1)
    assert c32.dtype == np.float32 and c32[0, 0] == 0.0
    assert abs(c64[0, 0] - 1.0 / 3.0) < 1e-15


def test_f32_definition_agrees_with_the_reading_away_from_ties():
    rng = np.random.default_rng(9)
    k = _mixture(rng, 1500, 32, 8, spread=5.0, noise=0.4)
    a32, c32 = M.kmeans_keys_f32(k, 12, 6)
    a64, c64 = M.kmeans_keys(k, 12, 6)
    assert np.array_equal(a32, a64)
    assert np.abs(c32 - c64).max() < 1e-5
    # exactly placed keys: identical, centroids exact
    C, L0 = 4, 64
    points = np.zeros((C, 8))
    points[np.arange(C), np.arange(C)] = 4.0
    lab = rng.integers(0, C, size=L0)
    lab[(np.arange(C) * L0) // C] = np.arange(C)
    kk = _bf(points[lab])
    a, c = M.kmeans_keys_f32(kk, C, 2)
    assert np.array_equal(a, lab) and np.array_equal(c.astype(np.float64), points)
