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
from oracle import method as M
from tests.util import oracle_row

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# (workload, attention kernel): the automatic choice everywhere, and the tile pipeline
# forced on the ragged workload (whose rows end in partial blocks)
FULL = [(synth.BLOCK128K, 0), (synth.NVFP4_128K, 0), (synth.TOKEN32K, 0), (synth.RAGGED, 0),
        (synth.RAGGED, 1)]


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
