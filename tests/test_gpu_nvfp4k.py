"""The NVFP4 storage variant's attended keys ("Jet-QSparse ...", Full text): qs_gather_kv_nvfp4k
against the oracle, then dense attention over the gathered buffer.

Inputs: the small copy of the NVFP4 128K workload (two kept blocks per row), filled and
decoded one step through the validated path.

The bar:
  * gathered keys bit-exact against nvfp4_attended_keys_bf16 (kept blocks' stored BF16
    keys; elsewhere the dequantised, un-centred key rounded to BF16); values bit-exact;
    row lengths as in gather-then-attend;
  * dense attention over the gathered buffer within max-abs 2e-2 (BF16 output) of the
    oracle's attention over those keys, and within the derived per-row L2 bound of
    tests/util.py.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import method as M
from oracle import step as OS
from tests.util import check_attention, oracle_row, query_scale_all

pytestmark = pytest.mark.gpu


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_nvfp4_attended_keys_and_attention():
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import GatheredKV, workspace
    from tests.gpu_util import Filled, out_to_f64
    w = synth.small(synth.NVFP4_128K)
    inp = synth.Inputs(w)
    f = Filled(inp)
    _, sel, nsel = f.decode()
    gk = GatheredKV.allocate(f.layer, fill=float("nan"))
    qs.qs_gather_kv_nvfp4k(f.cfg, f.cache, sel, nsel, w.batch, gk.k, gk.v, gk.row_lens,
                           f.layer.ws)
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    P, d, G = gk.pages_per_seq, w.head_dim, w.group
    kd = gk.k.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.batch, P, w.n_kv_heads, 128, d)
    vd = gk.v.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.batch, P, w.n_kv_heads, 128, d)
    row_lens = gk.row_lens.cpu().numpy()
    sel_h, nsel_h = sel.cpu().numpy(), nsel.cpu().numpy()
    ws = workspace(qs.qs_dense_workspace_size(f.cfg, w.batch, gk.max_context))
    out = torch.full((w.batch, w.n_q_heads, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    qs.qs_dense_attn(f.cfg, gk.cache(), f.q, gk.row_lens, w.batch, out, ws)
    st = qs.qs_device_status(ws)
    assert st[0] == 0, f"device status {st}"
    out = out_to_f64(out)
    gq = query_scale_all(inp, Q=f.Q)
    for b in range(w.batch):
        L = int(inp.lens[b])
        for g in range(w.n_kv_heads):
            got_sel = sel_h[b, g, :nsel_h[b, g]]
            src, n = M.gather_blocks(got_sel, w.block_size, L)
            assert row_lens[b * w.n_kv_heads + g] == n, f"row ({b},{g}) length"
            row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
            r = oracle_row(inp, b, g, row=row, g_q=gq, sel_override=got_sel)
            codes, scales, _ = r["cache"]
            Kb = M.nvfp4_attended_keys_bf16(f.K[b, g, :L], codes, scales, inp.g_k,
                                            inp.mu[b, g], r["keep"], w.block_size, L)
            krow = kd[b, :, g].reshape(P * 128, d)
            vrow = vd[b, :, g].reshape(P * 128, d)
            assert np.array_equal(krow[:n], Kb[src[:n]]), f"row ({b},{g}) K"
            assert np.array_equal(vrow[:n], f.V[b, g, :L][src[:n]]), f"row ({b},{g}) V"
            toks = M.block_tokens(got_sel, w.block_size, L)
            Kd = F.bf16_to_f64(Kb)
            want = M.sparse_attention(F.bf16_to_f64(row[2]), Kd,
                                      OS.decode_v(row[1], w.v_dtype), toks, w.scale)
            check_attention(w, out[b, g * G:(g + 1) * G], want, row, toks, f"row ({b},{g})",
                            K=Kd)
