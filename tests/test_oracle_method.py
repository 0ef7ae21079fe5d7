"""Pins of the oracle's writer, scorer, selector and attention.

Each check is against something other than the oracle's own formula: identities that
reduce the method to a textbook result, brute-force enumeration, exact arithmetic, or
error bounds of IEEE float32.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import formats as F
from oracle import method as M


def _bf16(x):
    return F.f32_to_bf16_rne(np.asarray(x, dtype=np.float32))


# ---------------------------------------------------------------- writer (projected keys)

def test_proxy_identity_projection_is_exact():
    rng = np.random.default_rng(0)
    k = _bf16(rng.standard_normal((50, 16)) * 4)
    P = np.eye(16, dtype=np.float32)
    out = M.proxy_keys_f32(k, P)
    assert np.array_equal(out, F.bf16_to_f64(k).astype(np.float32))


def test_proxy_single_entry_projection():
    rng = np.random.default_rng(1)
    k = _bf16(rng.standard_normal((20, 8)))
    P = np.zeros((8, 3), dtype=np.float32)
    P[5, 2] = np.float32(0.3)
    out = M.proxy_keys_f32(k, P)
    assert np.all(out[:, :2] == 0)
    want = (F.bf16_to_f64(k)[:, 5].astype(np.float32) * np.float32(0.3)).astype(np.float32)
    assert np.array_equal(out[:, 2], want)


def test_proxy_summation_order_is_ascending():
    # 2^24 + 1 is not a float32: adding in index order loses the 1, reversed order keeps it.
    k = _bf16(np.array([[2.0 ** 24, 1.0, -(2.0 ** 24)]]))
    P = np.ones((3, 1), dtype=np.float32)
    assert M.proxy_keys_f32(k, P)[0, 0] == 0.0


def test_proxy_rounds_each_product_before_adding():
    # The first term is -(1 + 2^-7 + 2^-23), exact. The second is (1 + 2^-7)(1 + 2^-23) =
    # 1 + 2^-7 + 2^-23 + 2^-30: rounded to float32 first, it cancels the first exactly; a
    # fused multiply-add onto the first would leave 2^-30.
    k = _bf16(np.array([[-1.0, 1.0 + 2.0 ** -7]]))
    assert F.bf16_to_f64(k)[0, 1] == 1.0 + 2.0 ** -7
    P = np.array([[1.0 + 2.0 ** -7 + 2.0 ** -23], [1.0 + 2.0 ** -23]], dtype=np.float32)
    assert float(P[0, 0]) == 1.0 + 2.0 ** -7 + 2.0 ** -23
    assert M.proxy_keys_f32(k, P)[0, 0] == 0.0


def test_proxy_float32_error_bound():
    rng = np.random.default_rng(2)
    d, r = 128, 32
    k = _bf16(rng.standard_normal((300, d)) * 3)
    P = rng.standard_normal((d, r)).astype(np.float32)
    kd = F.bf16_to_f64(k)
    exact = kd @ P.astype(np.float64)
    got = M.proxy_keys_f32(k, P).astype(np.float64)
    u = 2.0 ** -24
    gamma = d * u / (1 - d * u)
    bound = gamma * (np.abs(kd) @ np.abs(P.astype(np.float64)))
    assert np.all(np.abs(got - exact) <= bound)
    # and the bf16 store is the nearest-even rounding of that float32 value
    st = M.proxy_store(k, P, "bf16")
    assert np.all(np.abs(F.bf16_to_f64(st) - got) <= np.abs(got) * 2.0 ** -8 + 1e-38)


# ---------------------------------------------------------------- scoring

def test_group_mean_linearity():
    rng = np.random.default_rng(3)
    q = _bf16(rng.standard_normal((5, 64)))
    P = rng.standard_normal((64, 16)).astype(np.float32)
    per_head = F.bf16_to_f64(q) @ P.astype(np.float64)
    assert np.allclose(M.proxy_query(q, P), per_head.mean(axis=0), rtol=1e-13, atol=1e-13)


def test_full_rank_identity_equals_exact_group_mean_score():
    rng = np.random.default_rng(4)
    d, L = 32, 100
    q = _bf16(rng.standard_normal((4, d)))
    k = _bf16(rng.standard_normal((L, d)))
    P = np.eye(d, dtype=np.float32)
    s = M.token_scores(M.proxy_decode(M.proxy_store(k, P, "f32"), "f32"), M.proxy_query(q, P))
    qd, kd = F.bf16_to_f64(q), F.bf16_to_f64(k)
    for t in range(L):
        exact = math.fsum(sum(qd[h, i] for h in range(4)) / 4 * kd[t, i] for i in range(d))
        assert abs(s[t] - exact) <= 1e-12 * (1 + abs(exact))


def test_block_max_loops():
    rng = np.random.default_rng(5)
    for L, S in [(37, 8), (64, 16), (5, 1), (130, 64)]:
        s = rng.standard_normal(L)
        got = M.block_max(s, S)
        nb = (L + S - 1) // S
        assert got.shape == (nb,)
        for j in range(nb):
            assert got[j] == max(s[t] for t in range(j * S, min(L, (j + 1) * S)))
    s = rng.standard_normal(17)
    assert np.array_equal(M.block_max(s, 1), s)


# ---------------------------------------------------------------- selection

def _brute_select(beta, budget, forced):
    nb = len(beta)
    if nb <= budget:
        return list(range(nb))
    rest = [j for j in range(nb) if j not in set(forced)]
    need = budget - len(forced)

    def beats(a, b):  # a ranks before b
        return beta[a] > beta[b] or (beta[a] == beta[b] and a < b)

    winners = []
    for T in itertools.combinations(rest, need):
        out = [j for j in rest if j not in T]
        if all(beats(a, b) for a in T for b in out):
            winners.append(sorted(list(forced) + list(T)))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("seed", range(40))
def test_select_exhaustive(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(1, 11))
    budget = int(rng.integers(1, 9))
    beta = rng.integers(-3, 4, size=nb).astype(np.float64)      # many exact ties
    fs, fl = bool(rng.integers(0, 2)), bool(rng.integers(0, 2))
    forced = M.forced_blocks(nb, fs, fl)
    if nb > budget and len(forced) > budget:
        return
    got = M.select_blocks(beta, budget, forced)
    assert got.tolist() == _brute_select(beta, budget, forced.tolist())


def test_select_invariants():
    rng = np.random.default_rng(7)
    beta = rng.standard_normal(1000)
    forced = M.forced_blocks(1000, True, True)
    sel = M.select_blocks(beta, 64, forced)
    assert len(sel) == 64 and {0, 999} <= set(sel.tolist())
    chosen = np.setdiff1d(sel, forced)
    rest = np.setdiff1d(np.setdiff1d(np.arange(1000), sel), forced)
    assert beta[chosen].min() >= beta[rest].max()
    assert np.all(np.diff(sel) > 0)
    assert M.select_blocks(beta[:50], 64, forced[:1]).tolist() == list(range(50))


def test_selection_validity_rule():
    beta = np.array([5.0, 4.0, 3.0, 3.00001, 1.0, 0.0])
    forced = np.array([], dtype=np.int64)
    ok, why = M.selection_valid(beta, 3, forced, np.array([0, 1, 3]))
    assert ok and why == "exact"
    ok, why = M.selection_valid(beta, 3, forced, np.array([0, 1, 2]))   # within 1e-4 rel
    assert ok and why.startswith("near-tie")
    ok, _ = M.selection_valid(beta, 3, forced, np.array([0, 1, 4]))
    assert not ok
    ok, _ = M.selection_valid(beta, 3, forced, np.array([0, 1]))
    assert not ok


# ---------------------------------------------------------------- attention

def _dense_attention_bruteforce(q, K, V, scale):
    G, d = q.shape
    out = np.zeros((G, d))
    for h in range(G):
        logits = [scale * math.fsum(q[h, i] * K[t, i] for i in range(d)) for t in range(len(K))]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = math.fsum(w)
        for i in range(d):
            out[h, i] = math.fsum(w[t] * V[t, i] for t in range(len(K))) / z
    return out


def test_budget_covering_all_blocks_is_dense_attention():
    rng = np.random.default_rng(8)
    G, d, L, S = 3, 16, 45, 8
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((L, d))
    V = rng.standard_normal((L, d))
    nb = (L + S - 1) // S
    sel = M.select_blocks(rng.standard_normal(nb), nb + 2, M.forced_blocks(nb, True, True))
    toks = M.block_tokens(sel, S, L)
    assert toks.tolist() == list(range(L))
    got = M.sparse_attention(q, K, V, toks, 0.25)
    assert np.allclose(got, _dense_attention_bruteforce(q, K, V, 0.25), rtol=1e-12, atol=1e-12)


def test_one_hot_selection_returns_value_row():
    rng = np.random.default_rng(9)
    q, K, V = rng.standard_normal((2, 8)), rng.standard_normal((30, 8)), rng.standard_normal((30, 8))
    got = M.sparse_attention(q, K, V, np.array([17]), 1.0)
    assert np.array_equal(got, np.broadcast_to(V[17], (2, 8)))


@pytest.mark.parametrize("nsplit", [1, 2, 5, 13])
def test_lse_combine_split_invariance(nsplit):
    rng = np.random.default_rng(10 + nsplit)
    G, d, T = 4, 32, 200
    q = rng.standard_normal((G, d)) * 2
    K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    toks = np.sort(rng.choice(T, 120, replace=False))
    cuts = np.sort(rng.choice(np.arange(1, len(toks)), nsplit - 1, replace=False)) if nsplit > 1 else []
    parts = np.split(toks, cuts)
    parts.append(np.zeros(0, dtype=np.int64))                 # an empty split is ignored
    st = [M.attention_partial(q, K, V, p, 0.3) for p in parts]
    got = M.lse_combine([s[0] for s in st], [s[1] for s in st], [s[2] for s in st])
    assert np.allclose(got, M.sparse_attention(q, K, V, toks, 0.3), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- full-KV and gather-then-attend

def test_dense_attention_matches_loop_softmax():
    rng = np.random.default_rng(21)
    G, d, L = 4, 16, 37
    q = rng.standard_normal((G, d)) * 2
    K = rng.standard_normal((L + 5, d))            # rows at or past L are not attended
    V = rng.standard_normal((L + 5, d))
    got = M.dense_attention(q, K, V, L, 0.3)
    assert np.allclose(got, _dense_attention_bruteforce(q, K[:L], V[:L], 0.3),
                       rtol=1e-12, atol=1e-12)


def test_dense_attention_closed_forms():
    rng = np.random.default_rng(22)
    V = rng.standard_normal((9, 8))
    q = rng.standard_normal((3, 8))
    # equal keys: uniform weights, the mean of the values
    K = np.tile(rng.standard_normal(8), (9, 1))
    assert np.allclose(M.dense_attention(q, K, V, 9, 1.0), np.broadcast_to(V.mean(0), (3, 8)),
                       rtol=1e-13, atol=1e-13)
    # scale 0: the mean of the values whatever the keys
    K = rng.standard_normal((9, 8))
    assert np.allclose(M.dense_attention(q, K, V, 9, 0.0), np.broadcast_to(V.mean(0), (3, 8)),
                       rtol=1e-13, atol=1e-13)
    # one token: its value row; no token: zeros
    assert np.array_equal(M.dense_attention(q, K, V, 1, 1.0), np.broadcast_to(V[0], (3, 8)))
    assert np.array_equal(M.dense_attention(q, K, V, 0, 1.0), np.zeros((3, 8)))
    # one logit far above the rest: that token's value (weight of the others < e^-700)
    K2 = np.zeros((9, 8))
    K2[4, 0] = 1.0
    q2 = np.zeros((1, 8))
    q2[0, 0] = 700.0
    assert np.allclose(M.dense_attention(q2, K2, V, 9, 1.0)[0], V[4], rtol=0, atol=1e-290)


def test_gather_blocks_hand_example():
    # S = 4, L = 14 (blocks 0..3, block 3 holds tokens 12, 13 only); selected 1, 3
    src, n = M.gather_blocks(np.array([1, 3]), 4, 14)
    assert src.tolist() == [4, 5, 6, 7, 12, 13, -1, -1]
    assert n == 6
    # the cut block not selected: every slot filled
    src, n = M.gather_blocks(np.array([0, 2]), 4, 14)
    assert src.tolist() == [0, 1, 2, 3, 8, 9, 10, 11] and n == 8
    # token level (S = 1): the selection itself
    src, n = M.gather_blocks(np.array([3, 9, 10]), 1, 11)
    assert src.tolist() == [3, 9, 10] and n == 3
    # nothing selected
    src, n = M.gather_blocks(np.zeros(0, dtype=np.int64), 8, 5)
    assert src.size == 0 and n == 0


@pytest.mark.parametrize("seed", range(12))
def test_gather_prefix_and_count(seed):
    rng = np.random.default_rng(100 + seed)
    S = int(rng.choice([1, 2, 8, 16]))
    L = int(rng.integers(1, 200))
    nb = -(-L // S)
    k = int(rng.integers(1, nb + 1))
    sel = np.sort(rng.choice(nb, k, replace=False))
    src, n = M.gather_blocks(sel, S, L)
    # filled slots are a prefix, their tokens are exactly the selected valid tokens
    assert np.all(src[:n] >= 0) and np.all(src[n:] == -1)
    assert src[:n].tolist() == M.block_tokens(sel, S, L).tolist()
    # count: every selected block is full except a selected last block cut by L
    assert n == sum(min(S, L - b * S) for b in sel)


@pytest.mark.parametrize("seed", range(6))
def test_gather_then_dense_equals_sparse_attention(seed):
    # attending densely over the gathered prefix is the sparse attention over the selection
    rng = np.random.default_rng(200 + seed)
    G, d, S, L = 3, 16, int(rng.choice([1, 4, 16])), int(rng.integers(20, 300))
    nb = -(-L // S)
    sel = np.sort(rng.choice(nb, min(nb, int(rng.integers(1, 12))), replace=False))
    q = rng.standard_normal((G, d))
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    src, n = M.gather_blocks(sel, S, L)
    Kg = np.where(src[:, None] >= 0, K[np.maximum(src, 0)], np.nan)
    Vg = np.where(src[:, None] >= 0, V[np.maximum(src, 0)], np.nan)
    got = M.dense_attention(q, Kg, Vg, n, 0.2)
    want = _dense_attention_bruteforce(q, K[M.block_tokens(sel, S, L)], V[M.block_tokens(sel, S, L)], 0.2)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_e4m3_proxy_store_exact_for_representable_keys():
    # P = I and keys that are E4M3 values: the FP8 cache holds the keys exactly
    rng = np.random.default_rng(30)
    vals = F.e4m3_value(np.array([c for c in range(256) if c & 0x7F != 0x7F]))
    k = rng.choice(vals, size=(40, 16))
    kb = F.f32_to_bf16_rne(k.astype(np.float32))
    assert np.array_equal(F.bf16_to_f64(kb), k)            # E4M3 values are BF16 values
    st = M.proxy_store(kb, np.eye(16, dtype=np.float32), "e4m3")
    assert st.dtype == np.uint8
    assert np.array_equal(M.proxy_decode(st, "e4m3"), k)


def test_e4m3_proxy_store_rounds_the_float32_projection():
    # each stored entry is the E4M3 value nearest the float32 projection (relative error at
    # most 2^-4 in the normal range, saturating at 448)
    rng = np.random.default_rng(31)
    kb = _bf16(rng.standard_normal((64, 32)) * 3)
    P = np.linalg.qr(rng.standard_normal((32, 16)))[0].astype(np.float32)
    f32 = M.proxy_keys_f32(kb, P).astype(np.float64)
    dec = M.proxy_decode(M.proxy_store(kb, P, "e4m3"), "e4m3")
    normal = np.abs(f32) >= 2.0 ** -6
    assert np.all(np.abs(dec - f32)[normal] <= np.abs(f32)[normal] * 2.0 ** -4)
    assert np.all(np.abs(dec - f32)[~normal] <= 2.0 ** -10)


# ---------------------------------------------------------------- JSSA-style basis (spectral)

def _bf(x):
    return F.f32_to_bf16_rne(np.asarray(x, dtype=np.float32))


def test_basis_diagonal_moments_pick_coordinate_axes():
    # independent coordinates with distinct variances: the basis is the axes of the r
    # largest normalised variances, in that order, each with entry +1
    rng = np.random.default_rng(40)
    d, r, n = 16, 4, 4096
    sq = np.linspace(1.0, 4.0, d)[rng.permutation(d)]
    sk = np.linspace(0.5, 2.0, d)[rng.permutation(d)]
    # sign-randomised columns with exact per-coordinate energy (a Hadamard-like design)
    signs = rng.choice([-1.0, 1.0], size=(n, d))
    q = _bf((signs * sq)[:, None, :] * np.ones((1, 2, 1)))
    k = _bf(rng.choice([-1.0, 1.0], size=(n, d)) * sk)
    Mx = M.calibration_moment(q, k)
    # the diagonal is exactly the normalised energies of the coordinates
    eq, ek = np.array(sq, dtype=np.float64) ** 2, np.array(sk, dtype=np.float64) ** 2
    assert np.allclose(np.diag(Mx), eq / eq.sum() + ek / ek.sum(), rtol=1e-2)
    P, w = M.spectral_basis(np.diag(np.diag(Mx)), r)
    want_axes = np.argsort(-np.diag(Mx), kind="stable")[:r]
    assert np.array_equal(np.argmax(np.abs(P), axis=0), want_axes)
    assert np.allclose(np.abs(P).max(axis=0), 1.0) and np.all(P.max(axis=0) > 0)


def test_basis_recovers_a_shared_subspace():
    # queries and keys confined to span(U): the basis spans U exactly
    rng = np.random.default_rng(41)
    d, r, n = 32, 6, 2000
    U = np.linalg.qr(rng.standard_normal((d, r)))[0]
    q = _bf((rng.standard_normal((n, 3, r)) * np.array([5, 4, 3, 2, 1.5, 1.0])) @ U.T)
    k = _bf((rng.standard_normal((n, r)) * np.array([1, 2, 3, 4, 5, 6])) @ U.T)
    P, w = M.jssa_basis(q, k, r)
    # BF16 rounding adds a small component outside span(U)
    assert np.linalg.norm(P - U @ (U.T @ P)) < 0.02
    assert np.allclose(P.T @ P, np.eye(r), atol=1e-12)


def test_basis_unit_trace_normalisation():
    # scaling all queries (or all keys) by a power of two changes neither M nor P
    rng = np.random.default_rng(42)
    d, r, n = 24, 5, 1500
    A = rng.standard_normal((d, d))
    q = _bf(rng.standard_normal((n, 2, d)) @ A.T)
    k = _bf(rng.standard_normal((n, d)) @ np.diag(np.linspace(0.2, 3, d)))
    P0, w0 = M.jssa_basis(q, k, r)
    qs = _bf(F.bf16_to_f64(q) * 64.0)
    ks = _bf(F.bf16_to_f64(k) * 2.0 ** -5)
    P1, w1 = M.jssa_basis(qs, ks, r)
    assert np.allclose(M.calibration_moment(q, k), M.calibration_moment(qs, ks), atol=1e-13)
    assert np.allclose(P0, P1, atol=1e-10) and np.allclose(w0, w1, atol=1e-13)


def test_basis_normalisation_balances_queries_and_keys():
    # keys 1000x larger than queries: raw moments would follow the keys alone; the
    # normalised moment weighs both, so the query direction stays in the basis
    rng = np.random.default_rng(43)
    d, n = 8, 4000
    e = np.eye(d)
    q = _bf((rng.standard_normal((n, 1, 1)) * 3.0) * e[0][None, None, :])     # queries along e0
    k = _bf(rng.standard_normal((n, 2)) * 1000.0 @ e[[1, 2]])                  # keys along e1, e2
    P, w = M.jssa_basis(q, k, 1)
    assert np.argmax(np.abs(P[:, 0])) == 0 and abs(P[0, 0] - 1.0) < 1e-12
    assert abs(w[0] - 1.0) < 1e-12                                             # tr-normalised


def test_basis_is_rotation_equivariant():
    rng = np.random.default_rng(44)
    d, r, n = 16, 4, 3000
    Q = rng.standard_normal((n, 2, d)) * np.linspace(3, 0.5, d)
    K = rng.standard_normal((n, d)) * np.linspace(0.5, 2, d)[::-1]
    R = np.linalg.qr(rng.standard_normal((d, d)))[0]
    P0, w0 = M.spectral_basis(M.calibration_moment(_bf(Q), _bf(K)), r)
    # rotating the exact moment (not the rounded inputs) rotates the eigenvectors
    Mx = M.calibration_moment(_bf(Q), _bf(K))
    P1, w1 = M.spectral_basis(R @ Mx @ R.T, r)
    assert np.allclose(w0, w1, atol=1e-12)
    assert np.allclose(np.abs((R @ P0).T @ P1), np.eye(r), atol=1e-8)


# ---------------------------------------------------------------- centroid scoring

def test_centroid_score_is_the_mean_token_score():
    # linearity: qbar . mean(k) = mean(qbar . k) over the block's valid tokens
    rng = np.random.default_rng(50)
    G, d, S, L = 3, 16, 8, 45                    # 6 blocks, the last holds 5 tokens
    kb = _bf(rng.standard_normal((L, d)))
    qb = _bf(rng.standard_normal((G, d)))
    sums = M.centroid_sums(kb, S, L)
    beta = M.centroid_block_scores(qb, sums, S, L)
    qbar = F.bf16_to_f64(qb).mean(axis=0)
    tok = F.bf16_to_f64(kb) @ qbar
    want = np.array([tok[j * S:min(L, (j + 1) * S)].mean() for j in range(6)])
    assert np.allclose(beta, want, rtol=1e-6, atol=1e-6)


def test_centroid_sums_in_token_order():
    # hand case in float32: a block's sum restarts at its first token; exact for small ints
    k = _bf(np.array([[1.0, -2.0], [3.0, 0.5], [4.0, 4.0], [-1.0, 1.0], [2.0, 2.0]]))
    sums = M.centroid_sums(k, 2, 5)
    assert sums.tolist() == [[4.0, -1.5], [3.0, 5.0], [2.0, 2.0]]
    beta = M.centroid_block_scores(_bf(np.array([[1.0, 1.0]])), sums, 2, 5)
    assert beta.tolist() == [2.5 / 2, 8.0 / 2, 4.0 / 1]


def test_centroid_sums_round_in_float32_sequence():
    # 1 + 2^-24 + 2^-24: sequential float32 adds lose both small terms
    k = _bf(np.array([[1.0], [2.0 ** -24], [2.0 ** -24]]))
    assert M.centroid_sums(k, 4, 3)[0, 0] == np.float32(1.0)
    # token-level blocks (S = 1): each sum is the key itself
    kk = _bf(np.random.default_rng(51).standard_normal((7, 4)))
    assert np.array_equal(M.centroid_sums(kk, 1, 7), F.bf16_to_f64(kk).astype(np.float32))


# ---------------------------------------------------------------- the per-row step

def test_step_decodes_fp16_values_as_fp16():
    # 0x3E00 is 1.5 as FP16 but 0.125 as the top half of a float32 (BF16)
    from oracle import step as OS
    bits = np.array([[0x3E00, 0xBC00]], dtype=np.uint16)            # 1.5, -1.0 in FP16
    assert OS.decode_v(bits, "f16").tolist() == [[1.5, -1.0]]
    assert OS.decode_v(bits, "bf16").tolist() == [[0.125, -0.0078125]]


def test_step_attends_over_an_accepted_override():
    """With sel_override, the output is attention over the override's tokens (checked by a
    brute-force softmax), not over the oracle's own selection."""
    from oracle import step as OS
    rng = np.random.default_rng(31)
    S, L, d, G = 8, 64, 16, 2
    k = _bf16(rng.standard_normal((L, d)))
    v = _bf16(rng.standard_normal((L, d)))
    q = _bf16(rng.standard_normal((G, d)))
    P = np.linalg.qr(rng.standard_normal((d, 8)))[0].astype(np.float32)
    p = OS.RowParams(S=S, budget=3, scale=0.25, proxy="f32", v_dtype="bf16")
    own = OS.decode_row(p, k, v, q, L, P=P)
    other = np.setdiff1d(np.arange(L // S), own["sel"])[:3]
    r = OS.decode_row(p, k, v, q, L, P=P, sel_override=other)
    toks = [t for j in other for t in range(j * S, j * S + S)]
    K, V, Q = F.bf16_to_f64(k), F.bf16_to_f64(v), F.bf16_to_f64(q)
    for h in range(G):
        x = [0.25 * math.fsum(Q[h] * K[t]) for t in toks]
        m = max(x)
        w = [math.exp(z - m) for z in x]
        want = [math.fsum(w[i] * V[t, c] for i, t in enumerate(toks)) / math.fsum(w)
                for c in range(d)]
        assert np.allclose(r["out"][h], want, rtol=1e-12, atol=1e-12)


def test_step_rank_r_scores_are_the_group_mean_scores():
    """Rank d with P = I and an FP32 proxy: the step's block scores are the block maxima of
    the exact group-mean scores (the mean of the heads, not their sum)."""
    from oracle import step as OS
    rng = np.random.default_rng(32)
    S, L, d, G = 4, 30, 16, 3
    k = _bf16(rng.standard_normal((L, d)))
    q = _bf16(rng.standard_normal((G, d)))
    p = OS.RowParams(S=S, budget=2, scale=0.25, proxy="f32", v_dtype="bf16")
    r = OS.decode_row(p, k, k, q, L, P=np.eye(d, dtype=np.float32))
    K, Q = F.bf16_to_f64(k), F.bf16_to_f64(q)
    qbar = [math.fsum(Q[:, i]) / G for i in range(d)]
    s = [math.fsum(qbar[i] * K[t, i] for i in range(d)) for t in range(L)]
    want = [max(s[j * S:min(L, (j + 1) * S)]) for j in range(-(-L // S))]
    assert np.allclose(r["beta"], want, rtol=0, atol=1e-5 * max(map(abs, want)))
