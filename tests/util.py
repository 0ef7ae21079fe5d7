"""Helpers shared by the tests: map a synthetic workload onto the oracle's row parameters."""
import numpy as np

import synth
from oracle import method as M
from oracle import step as OS


row_params = OS.row_params_of
top_p_params = OS.top_p_params_of


def oracle_row(inp: synth.Inputs, b: int, g: int, row=None, g_q=None, sel_override=None,
               keep_override=None):
    w = inp.w
    k, v, q = row if row is not None else inp.row(b, g)
    L = int(inp.lens[b])
    if w.proxy_dtype == "rabitq":
        return OS.decode_row_top_p(top_p_params(w), k, v, q, L, inp.P[g], inp.mu[b, g],
                                   inp.u[b, g], sel_override=sel_override)
    P = inp.P[g] if inp.P is not None else None
    mu = inp.mu[b, g] if inp.mu is not None else None
    return OS.decode_row(row_params(w), k, v, q, L, P=P, mu=mu, g_k=inp.g_k, g_q=g_q,
                         sel_override=sel_override, keep_override=keep_override)


def query_scale_all(inp: synth.Inputs, Q=None):
    """Per-step NVFP4 query scale over the whole q tensor of the workload."""
    w = inp.w
    if Q is None:
        qs = [inp.row(b, g)[2] for b in range(w.batch) for g in range(w.n_kv_heads)]
        Q = np.stack(qs)
    return M.query_scale(Q)


# ---- the attention output bound ------------------------------------------------------------
#
# The kernels compute logits and the online softmax in FP32 and round the softmax weights to
# the P.V operand format (BF16, or FP16 where the workload aggregates values in FP16) before
# the FP32-accumulated product, then round the output to its format. Against the float64
# oracle on the same selected tokens, per row (the group's G x d outputs):
#   * each weight p_t carries a relative rounding error |delta_t| <= u_p (unit roundoff of
#     the P format, 2^-8 BF16, 2^-11 FP16), the same delta_t for every dimension; whether
#     the kernel's denominator sums the rounded or the unrounded weights, the error of
#     o_i is sum_t delta_t p_t (v_ti or v_ti - o_i) / l, so its L2 norm over the row is
#     about u_p * A with A^2 = sum_h sum_i sum_t (p_ht (|v_ti| + |o_hi|))^2 (independent
#     roundings; with few dominant weights the largest is exactly 1 and is not rounded);
#     the bound takes 2 u_p A;
#   * FP16 weights below 2^-14 are subnormal: absolute error <= 2^-25 per weight, at most
#     2^-25 * sqrt(G) * (||V_T||_F + sqrt(T) max_h ||o_h||) over the row;
#   * the output rounding: at most u_o ||o|| (u_o = 2^-8 BF16, 2^-24 FP32);
#   * FP32 logits, exp and accumulation: about 1e-6 relative, covered by 1e-5 ||o||.
# On the small workloads a float32 emulation of the kernels' arithmetic (64-token chunks,
# running max) lands at 0.1-0.4 of this bound, while dropping any one selected block of the
# block-level workloads moves the output by 1.2-60 times the bound
# (tests/test_attention_bound.py).

U_ROUND = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11, "f32": 2.0 ** -24}


def decoded_row(w: synth.Workload, row):
    """(q [G][d], K [L][d], V [L][d]) of a row's stored bits, decoded to float64."""
    from oracle import formats as F
    k, v, q = row
    return F.bf16_to_f64(q), F.bf16_to_f64(k), OS.decode_v(v, w.v_dtype)


def attention_bound(q, K, V, tokens, scale, want, p_dtype: str, out_dtype: str) -> float:
    """Bound on ||o_gpu - o_oracle||_2 over one row's outputs (derivation above).

    q [G][d], K / V [L][d] decoded float64, tokens the attended positions, want [G][d] the
    oracle's output over those tokens."""
    tokens = np.asarray(tokens, dtype=np.int64)
    Kt, Vt = K[tokens], V[tokens]
    lg = scale * (q @ Kt.T)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    V2 = (Vt ** 2).sum(axis=1)                               # [T]
    cross = np.abs(Vt) @ np.abs(want).T                      # [T][G]
    O2 = (want ** 2).sum(axis=1)                             # [G]
    A = np.sqrt(((p ** 2) * (V2[None, :] + 2.0 * cross.T + O2[:, None])).sum())
    on = float(np.linalg.norm(want))
    bound = 2.0 * U_ROUND[p_dtype] * A + U_ROUND[out_dtype] * on + 1e-5 * on
    if p_dtype == "f16":
        G = q.shape[0]
        bound += 2.0 ** -25 * np.sqrt(G) * (np.sqrt(V2.sum()) + np.sqrt(len(tokens)) *
                                             np.sqrt(O2.max()))
    return float(bound)


def attention_error(w: synth.Workload, got, want, q, K, V, tokens):
    """None if one row's output passes, else the reason.

    Both bars apply: the stated one (max-abs 2e-2 for BF16 outputs, relative L2 1e-3 for
    FP32 outputs) and the derived L2 bound above, which a dropped or mis-weighted block
    exceeds."""
    got = np.asarray(got, dtype=np.float64)
    if not np.all(np.isfinite(got)):
        return "non-finite output"
    diff = float(np.linalg.norm(got - want))
    on = max(float(np.linalg.norm(want)), 1e-30)
    if w.out_dtype == "f32":
        if diff / on > 1e-3:
            return f"rel-L2 {diff / on:.3e} > 1e-3"
    else:
        err = float(np.abs(got - want).max())
        if err > 2e-2:
            return f"max-abs {err:.3e} > 2e-2"
    bound = attention_bound(q, K, V, tokens, w.scale, want, w.v_agg_dtype, w.out_dtype)
    if diff > bound:
        return f"L2 error {diff:.3e} > derived bound {bound:.3e} (rel {diff / on:.3e})"
    return None


def check_attention(w: synth.Workload, got, want, row, tokens, where: str, K=None):
    """Assert one row's output against the oracle's over the same tokens. ``row`` is the
    row's stored bits (k, v, q); ``K`` replaces the decoded keys where the kernel attends
    other keys (the NVFP4 storage variant)."""
    q, Kd, Vd = decoded_row(w, row)
    if K is not None:
        Kd = K
    why = attention_error(w, got, want, q, Kd, Vd, tokens)
    assert why is None, f"{where}: {why}"


def attn_format(scale: float, v_agg_dtype: str = "bf16", out_dtype: str = "bf16"):
    """The three fields attention_error reads, for tests that build their own configuration
    instead of a synthetic workload (the library's defaults: BF16 P.V, BF16 output)."""
    from types import SimpleNamespace
    return SimpleNamespace(scale=scale, v_agg_dtype=v_agg_dtype, out_dtype=out_dtype)


def each_row(check, rows, threads: int | None = None):
    """Run check(b, g) -> None | reason for every row in a host thread pool (numpy releases
    the GIL; BLAS pinned to one thread per worker) and return the failures as strings."""
    import concurrent.futures as cf
    import os

    from threadpoolctl import threadpool_limits
    threads = threads or len(os.sched_getaffinity(0))

    def one(bg):
        try:
            why = check(*bg)
        except AssertionError as e:
            why = str(e) or "assertion"
        return None if why is None else f"row {bg}: {why}"

    with threadpool_limits(1), cf.ThreadPoolExecutor(threads) as ex:
        return [x for x in ex.map(one, rows) if x is not None]
