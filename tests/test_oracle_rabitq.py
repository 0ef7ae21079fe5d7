"""Pins of the oracle's binary proxy (RaBitQ codes of the keys, a 4-bit code of the query)
and of its top-p budget, against facts fixed outside the oracle:
- a rotated case built from exact dyadic numbers, where the 1-bit code loses nothing and the
  estimate must equal the exact score;
- unbiasedness over uniformly random rotations and query roundings (the estimator's
  published property), with a planted normalisation mistake that the same check catches;
- identity and signed-permutation rotations, hand-derived query codes, the packed layout;
- top-p by exhaustive subset search, closed forms for uniform and geometric masses, the
  budget cap, forced blocks, ties, and the validity check's verdicts.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import formats as F
from oracle import method as M
from oracle import step as ST


def _bf(x):
    return F.f32_to_bf16_rne(np.asarray(x, dtype=np.float32))


def _hadamard(n):
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def _signed_hadamard_rotation(rng, d):
    """(signs) H (permutation) (signs) / sqrt(d): orthogonal, entries +-1/sqrt(d), exact in
    float32 for d = 16, and not symmetric."""
    H = _hadamard(d)
    perm = rng.permutation(d)
    R = (rng.choice([-1.0, 1.0], size=d)[:, None] * H[:, perm]
         * rng.choice([-1.0, 1.0], size=d)[None, :]) / math.sqrt(d)
    assert np.array_equal(R @ R.T, np.eye(d)) and not np.array_equal(R, R.T)
    return R.astype(np.float32)


def _haar(rng, d):
    A = rng.standard_normal((d, d))
    Q, Rq = np.linalg.qr(A)
    return (Q * np.sign(np.diag(Rq))[None, :]).astype(np.float32)


# ---- the exactly representable rotated case -----------------------------------------------

def test_estimate_is_exact_when_the_rotated_residual_is_a_sign_vector():
    """Keys whose rotated residual is a * s (s a sign vector) lose nothing to the 1-bit
    code; a query whose rotated entries lie on the 4-bit grid loses nothing to its code.
    The estimate is then the exact score q_bar . k, for any rounding draws u < 1."""
    rng = np.random.default_rng(11)
    d, G = 16, 2
    R = _signed_hadamard_rotation(rng, d)
    R64 = R.astype(np.float64)
    c = rng.integers(-8, 9, size=d) / 4.0                      # quarters in [-2, 2]
    a = np.array([1.0, 2.0, 0.5, 1.0, 2.0, 1.0, 0.5, 1.0])
    s = rng.choice([-1.0, 1.0], size=(len(a), d))
    o = (a[:, None] * s) @ R64.T                               # o R = a s exactly
    k = c[None, :] + o
    k_bits = _bf(k)
    assert np.array_equal(F.bf16_to_f64(k_bits), k)            # dyadic, exact in BF16
    n = rng.integers(0, 16, size=d)
    n[rng.choice(d, size=2, replace=False)] = [0, 15]         # v_l = -1, v_r = 0.875
    qr = -1.0 + n / 8.0                                        # Delta = 1/8
    qbar = qr @ R64.T
    delta_h = rng.integers(-1, 2, size=d) / 4.0
    q = np.stack([qbar + delta_h, qbar - delta_h])            # group mean is qbar exactly
    q_bits = _bf(q)
    assert np.array_equal(F.bf16_to_f64(q_bits), q)

    bits, g = M.rabitq_encode(k_bits, R, c.astype(np.float32))
    assert np.array_equal(bits, (s > 0).astype(np.uint8))
    assert np.array_equal(g.astype(np.float64), a)             # |o|^2 / |y|_1 = a
    for u in (np.zeros(d), np.full(d, 0.5), np.full(d, 0.999)):
        codes, delta, vl, qb = M.rabitq_query(q_bits, R, u.astype(np.float32))
        assert np.array_equal(codes, n) and delta == np.float32(0.125) and vl == -1.0
        assert np.array_equal(qb.astype(np.float64), qbar)
        est = M.rabitq_scores(bits, g, codes, delta, vl, c, qb)
        assert np.allclose(est, k @ qbar, rtol=0, atol=1e-12), (est, k @ qbar)


# ---- unbiasedness over random rotations -----------------------------------------------------

def _mean_estimate(rng, encode, trials, d=32):
    k = rng.standard_normal(d).astype(np.float32) * 1.5
    c = (rng.standard_normal(d) * 0.5).astype(np.float32)
    k_bits = _bf(k[None, :])
    kf = F.bf16_to_f64(k_bits)[0]
    o = kf - c.astype(np.float64)
    q = o / np.linalg.norm(o) * 2.0 + rng.standard_normal((4, d)) * 0.7
    q_bits = _bf(q)
    ests = np.empty(trials)
    qbar = None
    for t in range(trials):
        R = _haar(rng, d)
        u = rng.random(d).astype(np.float32)
        bits, g = encode(k_bits, R, c)
        codes, delta, vl, qbar = M.rabitq_query(q_bits, R, u)
        ests[t] = M.rabitq_scores(bits, g, codes, delta, vl, c, qbar)[0]
    exact = float(kf @ qbar.astype(np.float64))
    return ests.mean(), ests.std(ddof=1) / math.sqrt(trials), exact


def test_estimate_is_unbiased_over_random_rotations():
    rng = np.random.default_rng(5)
    mean, se, exact = _mean_estimate(rng, M.rabitq_encode, 3000)
    assert abs(mean - exact) <= 5 * se, (mean, exact, se)
    assert se < 0.02 * abs(exact)                      # the check has the power to see 10 %


def test_unbiasedness_check_catches_a_dropped_normalisation():
    """Planted mistake: scale the signs by |o| / sqrt(d) (dropping the division by
    <x, y / |o|>, about 0.8 for random directions). The same check must reject it."""
    def encode_wrong(k_bits, R, c):
        bits, _ = M.rabitq_encode(k_bits, R, c)
        o = M.centre(k_bits, c).astype(np.float64)
        return bits, (np.linalg.norm(o, axis=1) / math.sqrt(o.shape[1])).astype(np.float32)

    rng = np.random.default_rng(5)
    mean, se, exact = _mean_estimate(rng, encode_wrong, 3000)
    assert abs(mean - exact) > 5 * se


# ---- special rotations, query codes, layout --------------------------------------------------

def test_identity_rotation_codes_are_the_signs_of_the_residual():
    rng = np.random.default_rng(3)
    d = 64
    k_bits = _bf(rng.standard_normal((20, d)))
    c = np.zeros(d, dtype=np.float32)
    bits, g = M.rabitq_encode(k_bits, np.eye(d, dtype=np.float32), c)
    kf = F.bf16_to_f64(k_bits)
    assert np.array_equal(bits, (kf > 0).astype(np.uint8))
    want = np.array([math.fsum(r * r) / math.fsum(np.abs(r)) for r in kf])
    assert np.allclose(g, want, rtol=2e-6, atol=0)


def test_signed_permutation_moves_and_flips_the_bits():
    rng = np.random.default_rng(4)
    d = 32
    k_bits = _bf(rng.standard_normal((12, d)))
    c = (rng.standard_normal(d) * 0.3).astype(np.float32)
    perm = rng.permutation(d)
    sg = rng.choice([-1.0, 1.0], size=d)
    R = np.zeros((d, d), dtype=np.float32)
    R[perm, np.arange(d)] = sg                       # y_i = sg_i o_perm(i)
    bits, g = M.rabitq_encode(k_bits, R, c)
    bits0, g0 = M.rabitq_encode(k_bits, np.eye(d, dtype=np.float32), c)
    o = M.centre(k_bits, c)
    y = o[:, perm] * sg[None, :]
    assert np.array_equal(bits, (y > 0).astype(np.uint8))
    assert np.allclose(g, g0, rtol=2e-6, atol=0)


def test_rotation_rounds_each_product_before_adding():
    """y_0 = -(1 + 2^-7 + 2^-23) + fp32((1 + 2^-7)(1 + 2^-23)) = 0 exactly, so its code bit
    is 0; a fused multiply-add would leave +2^-30 and set the bit."""
    k_bits = _bf(np.array([[-1.0, 1.0 + 2.0 ** -7]]))
    R = np.zeros((2, 2), dtype=np.float32)
    R[0, 0], R[1, 0] = 1.0 + 2.0 ** -7 + 2.0 ** -23, 1.0 + 2.0 ** -23
    R[0, 1] = 1.0
    bits, g = M.rabitq_encode(k_bits, R, np.zeros(2, dtype=np.float32))
    assert bits[0].tolist() == [0, 0]
    # |y|_1 = |y_1| = 1 and |o|^2 = 1 + (1 + 2^-7)^2 in float32
    assert g[0] == np.float32(np.float32(1.0) + np.float32((1.0 + 2.0 ** -7) ** 2))


def test_key_equal_to_the_centre_has_zero_factor():
    c = np.linspace(-1, 1, 16).astype(np.float32)
    k_bits = _bf(c[None, :])
    bits, g = M.rabitq_encode(k_bits, np.eye(16, dtype=np.float32), F.bf16_to_f64(k_bits)[0])
    assert g[0] == 0 and not bits.any()


def test_query_codes_by_hand():
    """R = I, one head: q' = q; v_l = -1, v_r = 0.875, Delta = 1/8, t = 8 (q - v_l)."""
    d = 16
    q = np.zeros(d)
    q[:6] = [-1.0, 0.875, 0.0, 0.0625, 0.0625, 0.5]
    u = np.full(d, 0.25, dtype=np.float32)
    u[3], u[4] = 0.5, 0.49
    codes, delta, vl, _ = M.rabitq_query(_bf(q[None, :]), np.eye(d, dtype=np.float32), u)
    assert delta == np.float32(0.125) and vl == np.float32(-1.0)
    # t: 0, 15, 8, 8.5, 8.5, 12; floor(t + u)
    assert codes[:6].tolist() == [0, 15, 8, 9, 8, 12]
    assert np.all(codes[6:] == 8)


def test_query_code_is_clamped_at_the_top_level():
    """t = 15 and u just below 1: 15 + u rounds to 16 in float32; the code stays 15."""
    d = 16
    q = np.zeros(d)
    q[0], q[1] = -1.0, 0.875
    u = np.zeros(d, dtype=np.float32)
    u[1] = np.nextafter(np.float32(1.0), np.float32(0.0))
    assert np.float32(np.float32(15.0) + u[1]) == np.float32(16.0)
    codes, *_ = M.rabitq_query(_bf(q[None, :]), np.eye(d, dtype=np.float32), u)
    assert codes[1] == 15


def test_constant_query_gives_zero_codes():
    d = 16
    q = np.full((3, d), 0.75)
    codes, delta, vl, _ = M.rabitq_query(_bf(q), np.eye(d, dtype=np.float32),
                                         np.full(d, 0.9, dtype=np.float32))
    assert delta == 0 and vl == np.float32(0.75) and not codes.any()


def test_packed_bits_layout():
    bits = np.zeros((2, 16), dtype=np.uint8)
    bits[0, [0, 7, 9]] = 1
    bits[1, [15]] = 1
    packed = M.rabitq_pack_bits(bits)
    assert packed.tolist() == [[0x81, 0x02], [0x00, 0x80]]
    rng = np.random.default_rng(0)
    b = rng.integers(0, 2, size=(5, 128)).astype(np.uint8)
    assert np.array_equal(M.rabitq_unpack_bits(M.rabitq_pack_bits(b), 128), b)


# ---- weights and masses ---------------------------------------------------------------------

def test_estimated_weights_are_a_softmax():
    rng = np.random.default_rng(8)
    s = rng.standard_normal(50) * 20
    w = M.estimated_weights(s, 0.125)
    e = [math.exp(0.125 * x - 0.125 * s.max()) for x in s]
    z = math.fsum(e)
    assert np.allclose(w, np.array(e) / z, rtol=1e-13, atol=0)
    assert np.allclose(M.estimated_weights(s + 1000.0, 0.125), w, rtol=1e-9, atol=0)


def test_block_mass_sums_valid_tokens():
    w = np.arange(1, 11, dtype=np.float64)
    assert M.block_mass(w, 4).tolist() == [10.0, 26.0, 19.0]
    assert M.block_mass(w, 1).tolist() == w.tolist()


# ---- top-p ----------------------------------------------------------------------------------

def _brute_top_p(mass, p, budget, forced):
    nb = len(mass)
    goal = p * mass.sum()
    F_ = set(int(j) for j in forced)
    best_set = None
    for k in range(len(F_), budget + 1):
        best, best_set = -1.0, None
        for comb in itertools.combinations(range(nb), k):
            if not F_ <= set(comb):
                continue
            m = sum(mass[list(comb)])
            if m > best:
                best, best_set = m, comb
        if best_set is not None and best >= goal:
            return sorted(best_set)
    return sorted(best_set)


def test_top_p_matches_exhaustive_search():
    rng = np.random.default_rng(21)
    for _ in range(400):
        nb = int(rng.integers(1, 8))
        mass = rng.random(nb) ** 3 + 1e-3
        mass /= mass.sum()
        nf = int(rng.integers(0, min(2, nb) + 1))
        forced = np.sort(rng.choice(nb, size=nf, replace=False))
        budget = int(rng.integers(max(1, nf), nb + 1))
        p = float(rng.uniform(0.05, 1.0))
        got = M.select_top_p(mass, p, budget, forced)
        assert got.tolist() == _brute_top_p(mass, p, budget, forced), (mass, p, budget, forced)
        assert M.top_p_valid(mass, p, budget, forced, got)[0]


def test_top_p_uniform_masses_take_ceil_p_n():
    nb = 100
    mass = np.full(nb, 0.01)
    for p, k in ((0.374, 38), (0.05, 5), (0.999, 100), (0.0001, 1)):
        got = M.select_top_p(mass, p, nb, np.zeros(0))
        assert got.tolist() == list(range(k)), p     # equal masses: lowest indices first


def test_top_p_geometric_masses_closed_form():
    rng = np.random.default_rng(2)
    rho, nb = 0.9, 200
    pos = rng.permutation(nb)
    mass = np.empty(nb)
    mass[pos] = rho ** np.arange(nb)                 # pos[i] holds the i-th largest
    for p in (0.8, 0.5, 0.95):
        total = (1 - rho ** nb) / (1 - rho)
        k = math.ceil(math.log(1 - p * total * (1 - rho)) / math.log(rho))
        got = M.select_top_p(mass, p, nb, np.zeros(0))
        assert got.tolist() == sorted(pos[:k].tolist()), p


def test_top_p_goal_reached_exactly_stops():
    """Dyadic masses sum exactly: a set whose mass equals p * total reaches the goal, so
    nothing more is taken ("reaches" is >=, the fewest blocks)."""
    mass = np.array([0.125, 0.5, 0.125, 0.25])
    assert M.select_top_p(mass, 0.75, 4, np.zeros(0)).tolist() == [1, 3]
    assert M.select_top_p(mass, 0.5, 4, np.zeros(0)).tolist() == [1]
    assert M.select_top_p(np.full(4, 0.25), 0.5, 4, np.zeros(0)).tolist() == [0, 1]
    assert M.select_top_p(mass, 1.0, 4, np.zeros(0)).tolist() == [0, 1, 2, 3]


def test_top_p_budget_caps_and_forced_blocks_count():
    mass = np.array([0.01, 0.3, 0.05, 0.2, 0.25, 0.04, 0.15])
    assert M.select_top_p(mass, 0.99, 3, np.zeros(0)).tolist() == [1, 3, 4]
    # forced light blocks are always in and their mass counts toward p
    assert M.select_top_p(mass, 0.5, 7, np.array([0, 6])).tolist() == [0, 1, 4, 6]
    # a forced set already past the goal takes nothing else
    assert M.select_top_p(mass, 0.5, 7, np.array([1, 4])).tolist() == [1, 4]
    with pytest.raises(ValueError):
        M.select_top_p(mass, 0.0, 3, np.zeros(0))
    with pytest.raises(ValueError):
        M.select_top_p(mass, 0.5, 1, np.array([0, 6]))


def test_top_p_validity_verdicts():
    rng = np.random.default_rng(9)
    mass = rng.random(40) ** 2
    forced = np.array([0, 39])
    want = M.select_top_p(mass, 0.6, 30, forced)
    assert M.top_p_valid(mass, 0.6, 30, forced, want)[0]
    extra = np.setdiff1d(np.arange(40), want)
    heavy_out = extra[np.argmax(mass[extra])]
    light_in = np.setdiff1d(want, forced)[np.argmin(mass[np.setdiff1d(want, forced)])]
    bad = {
        "short": np.setdiff1d(want, [light_in]),
        "not minimal": np.sort(np.append(want, heavy_out)),
        "swap": np.sort(np.append(np.setdiff1d(want, [np.setdiff1d(want, forced)[
            np.argmax(mass[np.setdiff1d(want, forced)])]]), heavy_out)),
        "forced": np.setdiff1d(want, [0]),
        "order": want[::-1],
    }
    for name, got in bad.items():
        assert not M.top_p_valid(mass, 0.6, 30, forced, got)[0], name
    # at the cap: the heaviest budget blocks are valid although the goal is not reached
    cap = M.select_top_p(mass, 0.99, 5, forced)
    assert len(cap) == 5 and M.top_p_valid(mass, 0.99, 5, forced, cap)[0]


# ---- the step ------------------------------------------------------------------------------

def test_step_selects_a_planted_block_and_attends_exactly():
    """A block whose keys align with the query carries most of the true attention; the
    binary proxy's top-p set holds it, and the output is exact attention over the set."""
    rng = np.random.default_rng(17)
    d, G, S, L = 128, 4, 16, 16 * 40 + 5
    R = _haar(rng, d)
    k = rng.standard_normal((L, d))
    m = rng.standard_normal(d)
    m /= np.linalg.norm(m)
    plant = 23
    k[plant * S:(plant + 1) * S] += 4.0 * m
    k_bits = _bf(k)
    v_bits = _bf(rng.standard_normal((L, d)))
    q_bits = _bf(3.0 * m[None, :] + 0.3 * rng.standard_normal((G, d)))
    c = F.bf16_to_f64(k_bits).mean(axis=0).astype(np.float32)
    u = rng.random(d).astype(np.float32)
    p = ST.TopPParams(S=S, p=0.5, budget=12, scale=1.0 / math.sqrt(d), v_dtype="bf16",
                      force_sink=True, force_last=True)
    r = ST.decode_row_top_p(p, k_bits, v_bits, q_bits, L, R, c, u)
    nb = -(-L // S)
    assert {plant, 0, nb - 1} <= set(r["sel"].tolist())
    assert M.top_p_valid(r["mass"], 0.5, 12, r["forced"], r["sel"])[0]
    q = F.bf16_to_f64(q_bits)
    K, V = F.bf16_to_f64(k_bits), F.bf16_to_f64(v_bits)
    toks = M.block_tokens(r["sel"], S, L)
    x = q @ K[toks].T / math.sqrt(d)
    e = np.exp(x - x.max(axis=1, keepdims=True))
    assert np.allclose(r["out"], (e @ V[toks]) / e.sum(axis=1, keepdims=True), rtol=1e-12,
                       atol=1e-12)


def test_step_weights_use_the_softmax_scale():
    """The top-p step's estimated weights are softmax(scale * score), recomputed here with
    math.fsum from the step's own scores; at another scale they differ."""
    rng = np.random.default_rng(23)
    d, G, S, L = 32, 2, 4, 90
    k_bits = _bf(rng.standard_normal((L, d)) * 2)
    v_bits = _bf(rng.standard_normal((L, d)))
    q_bits = _bf(rng.standard_normal((G, d)) * 2)
    R = _haar(rng, d)
    c = np.zeros(d, dtype=np.float32)
    u = rng.random(d).astype(np.float32)
    p = ST.TopPParams(S=S, p=0.7, budget=10, scale=0.3, v_dtype="bf16")
    r = ST.decode_row_top_p(p, k_bits, v_bits, q_bits, L, R, c, u)
    x = [0.3 * s for s in r["scores"]]
    m = max(x)
    e = [math.exp(z - m) for z in x]
    z = math.fsum(e)
    assert np.allclose(r["weights"], np.array(e) / z, rtol=1e-12, atol=0)
    assert not np.allclose(M.estimated_weights(r["scores"], 1.0), r["weights"], rtol=1e-3)
