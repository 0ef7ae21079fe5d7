"""The oracle on the synthetic workloads: planted-needle invariant, structural invariants,
dense reduction, and the generator's determinism."""
import numpy as np
import pytest

import synth
from synth import gen
from oracle import method as M
from tests.util import oracle_row, query_scale_all


def test_needle_block_is_selected():
    inp = synth.Inputs(synth.TINY_NEEDLE)
    r = oracle_row(inp, 0, 0)
    assert 37 in r["sel"].tolist()
    assert len(r["sel"]) == 8


def test_literal_tiny_runs(capsys):
    inp = synth.Inputs(synth.TINY)
    r = oracle_row(inp, 0, 0)
    assert len(r["sel"]) == 8 and r["out"].shape == (4, 64)
    print("literal tiny workload: needle block 37 selected =", 37 in r["sel"].tolist())


@pytest.mark.parametrize("w", [synth.small(w) for w in synth.ORDER[1:] + synth.VARIANTS],
                         ids=lambda w: w.name)
def test_small_workload_invariants(w):
    inp = synth.Inputs(w)
    gq = query_scale_all(inp) if w.proxy_dtype == "nvfp4" else None
    for b in range(w.batch):
        for g in (0, w.n_kv_heads - 1):
            r = oracle_row(inp, b, g, g_q=gq)
            L = int(inp.lens[b])
            nb = (L + w.block_size - 1) // w.block_size
            sel = r["sel"]
            if w.top_p > 0:
                assert 1 <= len(sel) <= w.budget
                assert M.top_p_valid(r["mass"], float(np.float32(w.top_p)), w.budget,
                                     r["forced"], sel)[0]
            else:
                assert len(sel) == min(w.budget, nb)
            assert set(r["forced"].tolist()) <= set(sel.tolist())
            if w.force_sink:
                assert sel[0] == 0
            if w.force_last:
                assert sel[-1] == nb - 1
            if w.n_keep_hp:
                assert len(r["keep"]) == min(w.n_keep_hp, L // w.block_size)
            if nb <= w.budget and w.top_p == 0:
                # budget covers every block: exactly dense attention
                assert r["tokens"].tolist() == list(range(L))
            assert np.all(np.isfinite(r["out"]))


def test_ragged_rows_with_budget_over_blocks_are_dense():
    lens = gen.lengths(synth.RAGGED)
    nb = (lens + 63) // 64
    assert lens.tolist()[29:] == [100, 1000, 2047]
    assert np.all(nb[29:] <= 32) and np.all(nb[:29] > 32)
    assert np.all(lens[:29] % 64 != 0) and lens[:29].min() >= 4096 and lens[:29].max() <= 131072


def test_generator_is_deterministic_and_prefix_stable():
    w = synth.small(synth.BLOCK128K)
    k1, v1 = gen.row_kv(w, 1, 3, 500)
    k2, v2 = gen.row_kv(w, 1, 3, 500)
    k3, _ = gen.row_kv(w, 1, 3, 200)
    assert np.array_equal(k1, k2) and np.array_equal(v1, v2) and np.array_equal(k1[:200], k3)
    pt, n = gen.page_table(w, gen.lengths(w))
    used = pt[pt >= 0]
    assert sorted(used.tolist()) == list(range(n))


def test_projection_is_orthonormal():
    P = gen.proj_matrix(synth.BLOCK128K)
    assert P.shape == (8, 128, 32)
    assert np.allclose(P[0].T.astype(np.float64) @ P[0], np.eye(32), atol=1e-6)
    assert np.array_equal(P[0], P[7])


def test_semantic_workload_rows():
    """The semantic workload's small copy through the oracle's semantic step: C = ceil(L0/S)
    clusters, min(budget, C) selected, every token after the prompt attended, finite
    outputs."""
    from oracle import step as OS
    w = synth.small(synth.SEMANTIC_128K)
    inp = synth.Inputs(w)
    p = OS.SemanticParams(S=w.block_size, budget=w.budget, iters=2, scale=w.scale,
                          v_dtype=w.v_dtype)
    for b in range(w.batch):
        L = int(inp.lens[b])
        L0 = L - 1
        k, v, q = inp.row(b, 0)
        r = OS.decode_row_semantic(p, k, v, q, L0, L)
        C = -(-L0 // w.block_size)
        assert r["centroids"].shape[0] == C and len(r["sel"]) == min(w.budget, C)
        assert L0 in r["tokens"].tolist() and np.all(np.diff(r["tokens"]) > 0)
        assert np.all(np.isfinite(r["out"]))
