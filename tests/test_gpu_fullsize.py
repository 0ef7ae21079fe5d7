"""Parity at the full workload sizes, in the launch configuration the bench times.

The whole step runs through qs_decode on the full batch, then qs_score once more on the
completed caches. The oracle recomputes EVERY row (sequence, KV head) one by one, in a
host thread pool, and each row must meet the small-size bar:
  * the scoring cache bit-exact (projected keys, NVFP4 codes and scales, centroid sums);
  * block scores within 2e-5 (rank-r, centroid) or 1e-4 (NVFP4) of the row's largest |beta|;
  * the selection a valid top-k under the oracle's scores (identical up to the 1e-4 near-tie
    rule), n_sel = min(budget, blocks), ascending, padded with -1, forced blocks present;
  * the output within max-abs 2e-2 (BF16) of the oracle's attention over the GPU's
    selection, and within the per-row L2 bound derived from the rounding of the softmax
    weights and the output (tests/util.py), which a dropped or mis-weighted block exceeds.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import method as M
from tests.util import (attention_error, decoded_row, each_row, oracle_row, query_scale_all)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# (workload, attention kernel): the automatic choice everywhere, and the tile pipeline
# forced on the ragged workload (whose rows end in partial blocks)
FULL = [(synth.BLOCK128K, 0), (synth.NVFP4_128K, 0), (synth.TOKEN32K, 0), (synth.RAGGED, 0),
        (synth.RAGGED, 1), (synth.FP8_128K, 0), (synth.CENTROID_128K, 0), (synth.TOKEN128K, 0),
        (synth.NVFP4_STORE_128K, 0)]


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rows(w):
    return [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)]


@pytest.mark.parametrize("case", FULL, ids=lambda c: f"{c[0].name}-path{c[1]}")
def test_fullsize_every_row(case):
    _gpu()
    import score_then_select_b200 as qs
    from tests.gpu_util import Filled, out_to_f64
    w, path = case
    inp = synth.Inputs(w)
    f = Filled(inp, attn_path=path)
    out, sel, nsel = f.decode()
    lay = f.layer
    scores = torch.full((w.batch, w.n_kv_heads, lay.nb_stride), np.nan, dtype=torch.float32,
                        device="cuda")
    qs.qs_score(f.cfg, f.cache, f.q, f.P, w.batch, scores, lay.ws)
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    out, sel, nsel = out_to_f64(out), sel.cpu().numpy(), nsel.cpu().numpy()
    scores = scores.cpu().numpy()
    berr = lay.block_err.cpu().numpy() if lay.block_err is not None else None
    host = f.host_caches()
    gq = query_scale_all(inp, Q=f.Q) if w.proxy_dtype == "nvfp4" else None
    G = w.group
    stol = 1e-4 if w.proxy_dtype == "nvfp4" else 2e-5

    def check(b, g):
        L = int(inp.lens[b])
        nb = -(-L // w.block_size)
        row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
        r = oracle_row(inp, b, g, row=row, g_q=gq)
        cache = f.row_proxy(b, g, host=host)
        if w.proxy_dtype == "nvfp4":
            if not (np.array_equal(cache[0], r["cache"][0]) and
                    np.array_equal(cache[1], r["cache"][1])):
                return "NVFP4 codes or scales differ"
        elif not np.array_equal(cache, r["cache"]):
            return "scoring cache differs"
        beta = scores[b, g, :nb]
        tol = stol * max(np.abs(r["beta"]).max(), 1e-30)
        bad = np.nonzero(~(np.abs(beta - r["beta"]) <= tol))[0]
        if len(bad):
            return f"block scores {bad[:5]}"
        n = int(nsel[b, g])
        got = sel[b, g, :n]
        if n != min(w.budget, nb) or not np.all(sel[b, g, n:] == -1):
            return f"n_sel {n} or padding"
        if n and not (np.all(np.diff(got) > 0) and got[0] >= 0 and got[-1] < nb):
            return "selection not ascending and in range"
        forced = r["forced"]
        kept = None
        if w.n_keep_hp:
            nfull = L // w.block_size
            codes, scl, x32 = r["cache"]
            err_or = M.block_quant_error(x32, codes, scl, inp.g_k, w.block_size, L)[:nfull]
            if not np.allclose(berr[b, g, :nfull], err_or, rtol=1e-5, atol=0):
                return "block errors"
            kept = M.kept_blocks(berr[b, g, :nfull].astype(np.float64), w.n_keep_hp)
            okk, why = M.selection_valid(err_or, w.n_keep_hp, np.zeros(0, np.int64), kept)
            if not okk:
                return f"kept blocks {why}"
            forced = M.forced_blocks(nb, w.force_sink, w.force_last, kept)
        ok, why = M.selection_valid(r["beta"], w.budget, forced, got)
        if not ok:
            return f"selection {why}"
        q, K, V = decoded_row(w, row)
        if w.key_storage == "nvfp4":               # the storage variant's attended keys
            r = oracle_row(inp, b, g, row=row, g_q=gq, sel_override=got, keep_override=kept)
            K = r["K_att"]
        tokens = r["tokens"] if np.array_equal(got, r["sel"]) else \
            M.block_tokens(got, w.block_size, L)
        want = r["out"] if np.array_equal(got, r["sel"]) else \
            M.sparse_attention(q, K, V, tokens, w.scale)
        return attention_error(w, out[b, g * G:(g + 1) * G], want, q, K, V, tokens)

    bad = each_row(check, _rows(w))
    assert not bad, f"{w.name}: {len(bad)} rows fail, e.g. " + "; ".join(bad[:4])


@pytest.mark.parametrize("w", [synth.BLOCK128K, synth.TOKEN32K], ids=lambda w: w.name)
def test_fullsize_dense_and_gather_then_attend(w):
    """Full-KV attention and gather-then-attend at the full sizes, every row: the gathered
    length exact, and both outputs against the oracle (dense attention over the whole row;
    sparse attention over the GPU's selection) under the same bar as the sparse path."""
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import GatheredKV, workspace
    from tests.gpu_util import Filled, out_to_f64
    inp = synth.Inputs(w)
    f = Filled(inp)
    out_s, sel, nsel = f.decode()
    lay = f.layer
    ws_d = workspace(qs.qs_dense_workspace_size(f.cfg, w.batch, lay.max_context))
    out_d = torch.zeros_like(out_s)
    qs.qs_dense_attn(f.cfg, f.cache, f.q, None, w.batch, out_d, ws_d)
    gk = GatheredKV.allocate(lay)
    qs.qs_gather_kv(f.cfg, f.cache, sel, nsel, w.batch, gk.k, gk.v, gk.row_lens, lay.ws)
    ws_g = workspace(qs.qs_dense_workspace_size(f.cfg, w.batch, gk.max_context))
    out_g = torch.zeros_like(out_s)
    qs.qs_dense_attn(f.cfg, gk.cache(), f.q, gk.row_lens, w.batch, out_g, ws_g)
    for ws in (ws_d, ws_g, lay.ws):
        st = qs.qs_device_status(ws)
        assert st[0] == 0, f"device status {st}"
    out_d, out_g = out_to_f64(out_d), out_to_f64(out_g)
    sel, nsel = sel.cpu().numpy(), nsel.cpu().numpy()
    row_lens = gk.row_lens.cpu().numpy()
    G = w.group

    def check(b, g):
        L = int(inp.lens[b])
        got = sel[b, g, :nsel[b, g]]
        want_len = sum(min(w.block_size, L - int(j) * w.block_size) for j in got)
        if row_lens[b * w.n_kv_heads + g] != want_len:
            return "gathered length"
        row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
        q, K, V = decoded_row(w, row)
        full = np.arange(L)
        why = attention_error(w, out_d[b, g * G:(g + 1) * G],
                              M.dense_attention(q, K, V, L, w.scale), q, K, V, full)
        if why:
            return "full-KV: " + why
        tokens = M.block_tokens(got, w.block_size, L)
        why = attention_error(w, out_g[b, g * G:(g + 1) * G],
                              M.sparse_attention(q, K, V, tokens, w.scale), q, K, V, tokens)
        return None if why is None else "gather-then-attend: " + why

    bad = each_row(check, _rows(w))
    assert not bad, f"{w.name}: {len(bad)} rows fail, e.g. " + "; ".join(bad[:4])
