"""Parity at the full workload sizes, in the launch configuration the bench times.

The whole step runs through qs_decode on the full batch; the oracle then recomputes a few
sampled rows (sequence, KV head) one by one, and every row is checked for the properties
that hold at any size: n_sel = min(budget, blocks), strictly ascending selections, forced
blocks present, finite outputs and scores.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import method as M
from tests.util import oracle_row

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# (workload, attention kernel): the automatic choice everywhere, and the tile pipeline
# forced on the ragged workload (whose rows end in partial blocks)
FULL = [(synth.BLOCK128K, 0), (synth.NVFP4_128K, 0), (synth.TOKEN32K, 0), (synth.RAGGED, 0),
        (synth.RAGGED, 1), (synth.FP8_128K, 0), (synth.CENTROID_128K, 0), (synth.TOKEN128K, 0)]


def _check_all_rows(w, inp, sel, nsel, out, berr):
    G = w.group
    for b in range(w.batch):
        L = int(inp.lens[b])
        nb = -(-L // w.block_size)
        for g in range(w.n_kv_heads):
            n = int(nsel[b, g])
            assert n == min(w.budget, nb)
            got = sel[b, g, :n]
            assert np.all(np.diff(got) > 0) and got[0] >= 0 and got[-1] < nb
            assert np.all(sel[b, g, n:] == -1)
            if nb > w.budget:
                if w.force_sink:
                    assert got[0] == 0
                if w.force_last:
                    assert got[-1] == nb - 1
                if w.n_keep_hp:
                    nfull = L // w.block_size
                    kept = M.kept_blocks(berr[b, g, :nfull].astype(np.float64), w.n_keep_hp)
                    assert set(kept.tolist()) <= set(got.tolist())
            assert np.all(np.isfinite(out[b, g * G:(g + 1) * G]))


@pytest.mark.parametrize("case", FULL, ids=lambda c: f"{c[0].name}-path{c[1]}")
def test_fullsize_sampled_rows(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.gpu_util import Filled, out_to_f64
    from tests.util import query_scale_all
    w, path = case
    inp = synth.Inputs(w)
    f = Filled(inp, attn_path=path)
    out, sel, nsel = f.decode()
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    out, sel, nsel = out_to_f64(out), sel.cpu().numpy(), nsel.cpu().numpy()
    berr = f.layer.block_err.cpu().numpy() if f.layer.block_err is not None else None
    _check_all_rows(w, inp, sel, nsel, out, berr)
    gq = query_scale_all(inp, Q=f.Q) if w.proxy_dtype == "nvfp4" else None
    rng = np.random.default_rng(7)
    rows = [(0, 0), (w.batch - 1, w.n_kv_heads - 1),
            (int(rng.integers(w.batch)), int(rng.integers(w.n_kv_heads)))]
    G = w.group
    for b, g in rows:
        row = (f.K[b, g, :inp.lens[b]], f.V[b, g, :inp.lens[b]], f.Q[b, g * G:(g + 1) * G])
        r = oracle_row(inp, b, g, row=row, g_q=gq)
        where = f"{w.name} row ({b},{g})"
        n = int(nsel[b, g])
        got = sel[b, g, :n]
        forced = r["forced"]
        if w.n_keep_hp:
            L = int(inp.lens[b])
            nfull = L // w.block_size
            kept = M.kept_blocks(berr[b, g, :nfull].astype(np.float64), w.n_keep_hp)
            nb = -(-L // w.block_size)
            forced = M.forced_blocks(nb, w.force_sink, w.force_last, kept)
        ok, why = M.selection_valid(r["beta"], w.budget, forced, got)
        assert ok, f"{where}: selection {why}"
        rr = r if np.array_equal(got, r["sel"]) else oracle_row(inp, b, g, row=row, g_q=gq,
                                                                 sel_override=got)
        err = np.abs(out[b, g * G:(g + 1) * G] - rr["out"]).max()
        assert err <= 2e-2, f"{where}: max-abs {err}"


@pytest.mark.parametrize("w", [synth.BLOCK128K, synth.TOKEN32K], ids=lambda w: w.name)
def test_fullsize_dense_and_gather_then_attend(w):
    """Full-KV attention and gather-then-attend at the full sizes: every row's gathered
    length exact and every output finite; sampled rows against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
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
    assert np.all(np.isfinite(out_d)) and np.all(np.isfinite(out_g))
    sel, nsel = sel.cpu().numpy(), nsel.cpu().numpy()
    row_lens = gk.row_lens.cpu().numpy()
    for b in range(w.batch):
        L = int(inp.lens[b])
        for g in range(w.n_kv_heads):
            got = sel[b, g, :nsel[b, g]]
            want = sum(min(w.block_size, L - int(j) * w.block_size) for j in got)
            assert row_lens[b * w.n_kv_heads + g] == want, f"row ({b},{g}) gathered length"
    rng = np.random.default_rng(11)
    G = w.group
    for b, g in [(0, 0), (w.batch - 1, w.n_kv_heads - 1),
                 (int(rng.integers(w.batch)), int(rng.integers(w.n_kv_heads)))]:
        L = int(inp.lens[b])
        row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
        q = F.bf16_to_f64(row[2])
        K = F.bf16_to_f64(row[0])
        V = F.f16_to_f64(row[1]) if w.v_dtype == "f16" else F.bf16_to_f64(row[1])
        err = np.abs(out_d[b, g * G:(g + 1) * G] - M.dense_attention(q, K, V, L, w.scale)).max()
        assert err <= 2e-2, f"{w.name} row ({b},{g}) full-KV max-abs {err}"
        r = oracle_row(inp, b, g, row=row, sel_override=sel[b, g, :nsel[b, g]])
        err = np.abs(out_g[b, g * G:(g + 1) * G] - r["out"]).max()
        assert err <= 2e-2, f"{w.name} row ({b},{g}) gather-then-attend max-abs {err}"
