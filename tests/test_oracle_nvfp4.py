"""Pins of the oracle's NVFP4 path: packing, block-scaled dot products, block errors."""
import itertools
import math

import numpy as np
import pytest

from oracle import formats as F
from oracle import method as M


def test_exactly_representable_groups_round_trip():
    rng = np.random.default_rng(0)
    n, d = 40, 128
    codes = rng.integers(0, 16, size=(n, d)).astype(np.uint8)
    codes[:, ::16] = 7                       # a 6 in every group: group scale becomes 1.0
    x = F.e2m1_value(codes).astype(np.float32)
    c2, s2 = M.nvfp4_pack(x, np.float32(1.0))
    assert np.all(s2 == 0x38)
    # -0 and +0 both decode to 0; compare values, and codes where the value is non-zero
    assert np.array_equal(F.e2m1_value(c2), F.e2m1_value(codes))
    nz = F.e2m1_value(codes) != 0
    assert np.array_equal(c2[nz], codes[nz])


def test_zero_group_has_zero_scale_and_codes():
    x = np.zeros((2, 32), dtype=np.float32)
    x[1, 16:] = np.linspace(-1, 1, 16)
    c, s = M.nvfp4_pack(x, np.float32(0.01))
    assert s[0].tolist() == [0, 0] and s[1, 0] == 0
    assert np.all(c[0] == 0) and np.all(c[1, :16] == 0)


def test_scale_saturates():
    x = np.full((1, 16), 1e6, dtype=np.float32)
    c, s = M.nvfp4_pack(x, np.float32(1.0))
    assert s[0, 0] == 0x7E and np.all(c == 7)


def test_per_element_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((500, 128)) * rng.uniform(0.01, 5, size=(500, 1))).astype(np.float32)
    g = np.float32(np.abs(x).max() / 2688.0)
    codes, scales = M.nvfp4_pack(x, g)
    deq = M.nvfp4_dequant(codes, scales, g)
    sig = F.ue4m3_value(scales).repeat(16, axis=1) * float(g)
    # the E2M1 grid's largest half-gap is 1.0 (between 4 and 6) in units of sigma * g
    assert np.all(np.abs(x - deq) <= sig * 1.0 + 1e-30)
    rel = np.linalg.norm(x - deq) / np.linalg.norm(x)
    assert rel < 0.12


def test_factored_block_scaled_dot_equals_dequantised_dot():
    """g_q g_k sum_c sq_c sk_c sum_i eq_i ek_i, evaluated by loops, equals deq(q) . deq(k)."""
    rng = np.random.default_rng(2)
    q = (rng.standard_normal((3, 128)) * 2).astype(np.float32)
    k = rng.standard_normal((7, 128)).astype(np.float32)
    gq, gk = np.float32(0.0013), np.float32(0.0021)
    qc, qs = M.nvfp4_pack(q, gq)
    kc, ks = M.nvfp4_pack(k, gk)
    got = M.nvfp4_head_scores(qc, qs, gq, kc, ks, gk)
    for h in range(3):
        for t in range(7):
            terms = []
            for c in range(8):
                inner = sum(F.E2M1_MAG[qc[h, 16 * c + i] & 7] * (-1 if qc[h, 16 * c + i] & 8 else 1)
                            * F.E2M1_MAG[kc[t, 16 * c + i] & 7] * (-1 if kc[t, 16 * c + i] & 8 else 1)
                            for i in range(16))
                terms.append(float(F.ue4m3_value(qs[h, c])) * float(F.ue4m3_value(ks[t, c])) * inner)
            want = float(gq) * float(gk) * math.fsum(terms)
            assert abs(got[h, t] - want) <= 1e-12 * (1 + abs(want))


def test_block_scores_max_over_heads_and_tokens_loops():
    rng = np.random.default_rng(3)
    hs = rng.standard_normal((5, 300))
    got = M.nvfp4_block_scores(hs, 128)
    for j in range(3):
        want = max(hs[h, t] for h in range(5) for t in range(j * 128, min(300, j * 128 + 128)))
        assert got[j] == want


def test_block_error_exact_and_single_perturbation():
    S = 16
    codes = np.full((64, 32), 2, dtype=np.uint8)            # value 1.0
    codes[:, 0] = 7                                         # a 6 -> group scale 1.0
    codes[:, 16] = 7
    x = F.e2m1_value(codes).astype(np.float32)
    c, s = M.nvfp4_pack(x, np.float32(1.0))
    err = M.block_quant_error(x, c, s, np.float32(1.0), S, 64)
    assert np.all(err == 0)
    x2 = x.copy()
    x2[37, 5] = np.float32(1.2)                              # rounds to 1.0 -> error 0.04
    c2, s2 = M.nvfp4_pack(x2, np.float32(1.0))
    err2 = M.block_quant_error(x2, c2, s2, np.float32(1.0), S, 64)
    assert err2.tolist()[:2] == [0.0, 0.0] and err2[3] == 0.0
    assert abs(err2[2] - (float(np.float32(1.2)) - 1.0) ** 2) < 1e-15
    # the incomplete last block has no error
    err3 = M.block_quant_error(x2[:60], c2[:60], s2[:60], np.float32(1.0), S, 60)
    assert err3.shape == (4,) and err3[3] == -np.inf


@pytest.mark.parametrize("seed", range(20))
def test_kept_blocks_exhaustive(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(1, 9))
    err = rng.integers(0, 4, size=nb).astype(np.float64)
    if rng.integers(0, 2):
        err[-1] = -np.inf
    valid = [j for j in range(nb) if np.isfinite(err[j])]
    n = min(2, len(valid))
    best = None
    for T in itertools.combinations(valid, n):
        key = sorted([(-err[j], j) for j in T])
        if best is None or key < best[0]:
            best = (key, sorted(T))
    assert M.kept_blocks(err, 2).tolist() == best[1]


def test_query_scale():
    q = F.f32_to_bf16_rne(np.array([[0.5, -3.0], [2.0, 1.0]], dtype=np.float32))
    assert M.query_scale(q) == np.float32(np.float32(3.0) / np.float32(2688.0))


# ---------------------------------------------------------------- attending over NVFP4 keys

def _nvfp4_row(rng, L, d=128):
    kb = F.f32_to_bf16_rne(rng.standard_normal((L, d)).astype(np.float32) * 2)
    mu = rng.standard_normal(d).astype(np.float32) * 0.1
    x32 = M.centre(kb, mu)
    g_k = np.float32(np.abs(x32).max() / (6.0 * 448.0))
    codes, scales = M.nvfp4_pack(x32, g_k)
    return kb, mu, x32, g_k, codes, scales


def test_attended_keys_use_bf16_in_kept_blocks_only():
    rng = np.random.default_rng(60)
    S, L = 16, 70
    kb, mu, x32, g_k, codes, scales = _nvfp4_row(rng, L)
    K = M.nvfp4_attended_keys(kb, codes, scales, g_k, mu, [1, 4], S, L)
    bf = F.bf16_to_f64(kb)
    deq = M.nvfp4_dequant(codes, scales, g_k) + mu.astype(np.float64)
    for t in range(L):
        want = bf[t] if t // S in (1, 4) else deq[t]
        assert np.array_equal(K[t], want), t
    # the cut last block (4: tokens 64..69) is kept whole up to L
    assert np.array_equal(K[64:70], bf[64:70])


def test_attended_keys_all_kept_is_bf16_attention():
    rng = np.random.default_rng(61)
    S, L = 8, 40
    kb, mu, x32, g_k, codes, scales = _nvfp4_row(rng, L)
    K = M.nvfp4_attended_keys(kb, codes, scales, g_k, mu, range(5), S, L)
    assert np.array_equal(K, F.bf16_to_f64(kb))


def test_attended_keys_error_within_the_nvfp4_bound():
    # away from kept blocks each key differs from the float32 key by at most the per-element
    # NVFP4 bound: half the largest E2M1 step (2 at magnitude 4..6) times sigma * g_k, plus
    # the float32 rounding of the centring
    rng = np.random.default_rng(62)
    S, L, d = 16, 64, 128
    kb, mu, x32, g_k, codes, scales = _nvfp4_row(rng, L, d)
    K = M.nvfp4_attended_keys(kb, codes, scales, g_k, mu, [], S, L)
    sig = F.ue4m3_value(scales).repeat(16, axis=1) * np.float64(g_k)
    err = np.abs(K - F.bf16_to_f64(kb))
    assert np.all(err <= 1.0 * sig + 1e-6 * np.abs(F.bf16_to_f64(kb)) + 1e-7)


def test_attended_keys_bf16_round_the_float64_keys():
    """The BF16 form is the float64 keys rounded to BF16, up to the float32 steps before the
    rounding: within half a BF16 step (plus the float32 error) everywhere, and the stored
    bits in kept blocks."""
    rng = np.random.default_rng(63)
    S, L = 16, 70
    kb, mu, x32, g_k, codes, scales = _nvfp4_row(rng, L)
    K64 = M.nvfp4_attended_keys(kb, codes, scales, g_k, mu, [2], S, L)
    Kb = M.nvfp4_attended_keys_bf16(kb, codes, scales, g_k, mu, [2], S, L)
    assert Kb.dtype == np.uint16
    assert np.array_equal(Kb[32:48], kb[32:48])
    got = F.bf16_to_f64(Kb)
    half_ulp = np.abs(K64) * 2.0 ** -8
    assert np.all(np.abs(got - K64) <= half_ulp + np.abs(K64) * 2.0 ** -22 + 1e-30)


def test_attended_keys_bf16_exact_for_representable_values():
    """Codes of E2M1 values, unit scales, g_k a power of two and a zero centre: every step
    is exact, so the BF16 keys are the dequantised values themselves."""
    rng = np.random.default_rng(64)
    L, d = 20, 128
    codes = rng.integers(0, 16, size=(L, d)).astype(np.uint8)
    scales = np.full((L, d // 16), 0x38, dtype=np.uint8)            # UE4M3 1.0
    g_k = np.float32(0.25)
    kb = np.zeros((L, d), dtype=np.uint16)
    Kb = M.nvfp4_attended_keys_bf16(kb, codes, scales, g_k, np.zeros(d, np.float32), [], 16, L)
    assert np.array_equal(F.bf16_to_f64(Kb), F.e2m1_value(codes) * 0.25)


def test_attended_keys_bf16_round_half_to_even():
    """A dequantised value halfway between two BF16 neighbours rounds to the even one:
    e * sigma * g = 1 * 1 * (1 + 2^-8) is exactly between 1 and 1 + 2^-7."""
    L, d = 1, 128
    codes = np.zeros((L, d), dtype=np.uint8)
    codes[0, 0] = 2                                                  # E2M1 1.0
    scales = np.full((L, d // 16), 0x38, dtype=np.uint8)
    g_k = np.float32(1.0 + 2.0 ** -8)
    Kb = M.nvfp4_attended_keys_bf16(np.zeros((L, d), np.uint16), codes, scales, g_k,
                                    np.zeros(d, np.float32), [], 16, L)
    assert F.bf16_to_f64(Kb)[0, 0] == 1.0


def _nvfp4_step_row(rng, L=512, G=4, n_keep=2, budget=3):
    from oracle import step as OS
    d, S = 128, 128
    k = F.f32_to_bf16_rne((rng.standard_normal((L, d)) * 1.5 + 0.5).astype(np.float32))
    v = F.f32_to_bf16_rne(rng.standard_normal((L, d)).astype(np.float32))
    # queries 40x larger than the keys: their tensor scale differs from the keys' by as much
    q = F.f32_to_bf16_rne((rng.standard_normal((G, d)) * 80).astype(np.float32))
    mu = F.bf16_to_f64(k).mean(axis=0).astype(np.float32)
    g_k = np.float32(np.abs(M.centre(k, mu)).max() / np.float32(2688.0))
    g_q = M.query_scale(q)
    p = OS.RowParams(S=S, budget=budget, scale=1 / np.sqrt(d), proxy="nvfp4", v_dtype="bf16",
                     force_sink=False, force_last=False, n_keep=n_keep)
    r = OS.decode_row(p, k, v, q, L, mu=mu, g_k=g_k, g_q=g_q)
    return r, k, q, mu


def test_step_nvfp4_scores_approximate_the_exact_centred_scores():
    """The NVFP4 step's block scores (max over heads and tokens of the FP4 dot of the packed
    query and centred keys) are within a quarter of the largest exact score of
    max_h,t q_h . (k_t - mu): the query packed with its own tensor scale."""
    rng = np.random.default_rng(70)
    r, k, q, mu = _nvfp4_step_row(rng)
    x = F.bf16_to_f64(k) - mu.astype(np.float64)
    s = F.bf16_to_f64(q) @ x.T
    exact = s.max(axis=0).reshape(-1, 128).max(axis=1)
    assert np.abs(r["beta"] - exact).max() <= 0.25 * np.abs(exact).max()


def test_step_nvfp4_kept_blocks_are_forced_and_selected():
    rng = np.random.default_rng(71)
    r, *_ = _nvfp4_step_row(rng, L=1024, n_keep=2, budget=3)
    assert len(r["keep"]) == 2
    assert set(r["keep"].tolist()) <= set(r["forced"].tolist())
    assert set(r["keep"].tolist()) <= set(r["sel"].tolist())


def test_step_key_storage_attends_the_storage_keys():
    """With NVFP4 key storage the row step attends over nvfp4_attended_keys (the kept
    blocks' BF16 keys, elsewhere the exactly dequantised, un-centred keys), with the same
    selection; keeping every selected block gives exactly the BF16-key output."""
    import dataclasses
    from oracle import step as OS
    rng = np.random.default_rng(72)
    L, G, d, S = 1000, 4, 128, 128
    k = F.f32_to_bf16_rne((rng.standard_normal((L, d)) * 1.5 + 0.5).astype(np.float32))
    v = F.f32_to_bf16_rne(rng.standard_normal((L, d)).astype(np.float32))
    q = F.f32_to_bf16_rne((rng.standard_normal((G, d)) * 3).astype(np.float32))
    mu = F.bf16_to_f64(k).mean(axis=0).astype(np.float32)
    g_k = np.float32(np.abs(M.centre(k, mu)).max() / np.float32(2688.0))
    g_q = M.query_scale(q)
    p = OS.RowParams(S=S, budget=5, scale=1 / np.sqrt(d), proxy="nvfp4", v_dtype="bf16",
                     force_sink=True, force_last=True, n_keep=2)
    ps = dataclasses.replace(p, key_storage="nvfp4")
    r_bf = OS.decode_row(p, k, v, q, L, mu=mu, g_k=g_k, g_q=g_q)
    r_st = OS.decode_row(ps, k, v, q, L, mu=mu, g_k=g_k, g_q=g_q)
    assert np.array_equal(r_st["sel"], r_bf["sel"]) and len(r_st["keep"]) == 2
    codes, scales, _ = r_st["cache"]
    want_k = M.nvfp4_attended_keys(k, codes, scales, g_k, mu, r_st["keep"], S, L)
    assert np.array_equal(r_st["K_att"], want_k)
    Vd = OS.decode_v(v, p.v_dtype)
    assert np.array_equal(r_st["out"], M.sparse_attention(F.bf16_to_f64(q), want_k, Vd,
                                                          r_st["tokens"], p.scale))
    # the non-kept selected blocks are attended with their NVFP4 keys: the output moves
    assert not np.allclose(r_st["out"], r_bf["out"], rtol=1e-6, atol=0)
    r_all = OS.decode_row(ps, k, v, q, L, mu=mu, g_k=g_k, g_q=g_q, keep_override=r_st["sel"])
    assert np.array_equal(r_all["out"], r_bf["out"])
