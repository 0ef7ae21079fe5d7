"""Helpers shared by the tests: map a synthetic workload onto the oracle's row parameters."""
import numpy as np

import synth
from oracle import method as M
from oracle import step as OS


def row_params(w: synth.Workload) -> OS.RowParams:
    return OS.RowParams(S=w.block_size, budget=w.budget, scale=w.scale, proxy=w.proxy_dtype,
                        v_dtype=w.v_dtype, force_sink=w.force_sink, force_last=w.force_last,
                        n_keep=w.n_keep_hp)


def top_p_params(w: synth.Workload) -> OS.TopPParams:
    """The binary proxy's row parameters; p as the float32 the C ABI takes."""
    return OS.TopPParams(S=w.block_size, p=float(np.float32(w.top_p)), budget=w.budget,
                         scale=w.scale, v_dtype=w.v_dtype, force_sink=w.force_sink,
                         force_last=w.force_last)


def oracle_row(inp: synth.Inputs, b: int, g: int, row=None, g_q=None, sel_override=None):
    w = inp.w
    k, v, q = row if row is not None else inp.row(b, g)
    L = int(inp.lens[b])
    if w.proxy_dtype == "rabitq":
        return OS.decode_row_top_p(top_p_params(w), k, v, q, L, inp.P[g], inp.mu[b, g],
                                   inp.u[b, g], sel_override=sel_override)
    P = inp.P[g] if inp.P is not None else None
    mu = inp.mu[b, g] if inp.mu is not None else None
    return OS.decode_row(row_params(w), k, v, q, L, P=P, mu=mu, g_k=inp.g_k, g_q=g_q,
                         sel_override=sel_override)


def query_scale_all(inp: synth.Inputs, Q=None):
    """Per-step NVFP4 query scale over the whole q tensor of the workload."""
    w = inp.w
    if Q is None:
        qs = [inp.row(b, g)[2] for b in range(w.batch) for g in range(w.n_kv_heads)]
        Q = np.stack(qs)
    return M.query_scale(Q)
