"""Parity of the comparison kernels with the oracle: full-KV attention (qs_dense_attn) and
gather-then-attend (qs_gather_kv, then qs_dense_attn over the compact buffer).

"Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 2 (b) and
Figure 6 (a), compare sparse attention with both. The bar:
  * gathered K / V bit-exact against the oracle's gathered layout, gathered lengths exact,
    the slots after them untouched;
  * attention outputs as for the sparse path: max-abs <= 2e-2 (BF16 outputs), relative
    L2 <= 1e-3 (FP32 outputs), and the per-row L2 bound derived from the rounding of the
    softmax weights and the output (tests/util.py), against the oracle in float64.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import method as M
from oracle import step as OS
from tests.util import attention_error, oracle_row, query_scale_all

pytestmark = pytest.mark.gpu

WORKLOADS = [synth.TINY, synth.TINY_CENTROID] + [synth.small(w) for w in (
    synth.TOKEN32K, synth.BLOCK128K, synth.NVFP4_128K, synth.RAGGED)]


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check_out(w, got, want, q, K, V, tokens, where):
    why = attention_error(w, got, want, q, K, V, tokens)
    assert why is None, f"{where}: {why}"


def _decoded(f, b, g):
    """(q, K, V) of row (b, g) decoded to float64, and the K / V bits, from the host copy the
    layer was filled from."""
    w = f.w
    L, G = int(f.inp.lens[b]), w.group
    kb, vb, qb = f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G]
    return F.bf16_to_f64(qb), F.bf16_to_f64(kb), OS.decode_v(vb, w.v_dtype), kb, vb


def _out_tensor(w):
    dt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    return torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=dt, device="cuda")


def _dense(f, cache, row_lens, max_context):
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import workspace
    w = f.w
    ws = workspace(qs.qs_dense_workspace_size(f.cfg, w.batch, max_context))
    out = _out_tensor(w)
    qs.qs_dense_attn(f.cfg, cache, f.q, row_lens, w.batch, out, ws)
    st = qs.qs_device_status(ws)
    assert st[0] == 0, f"device status {st}"
    return out


@pytest.mark.parametrize("w", WORKLOADS + [synth.small(synth.NVFP4_STORE_128K)],
                         ids=lambda w: w.name)
def test_dense_full_kv(w):
    """Full-KV attention; under the NVFP4 storage configuration it still reads the BF16
    key pages (the comparison the pages make is with BF16 attention)."""
    _gpu()
    from tests.gpu_util import Filled, out_to_f64
    inp = synth.Inputs(w)
    f = Filled(inp)
    f.decode()                                      # the caches now hold every row's L tokens
    out = out_to_f64(_dense(f, f.cache, None, f.layer.max_context))
    G = w.group
    for b in range(w.batch):
        L = int(inp.lens[b])
        for g in range(w.n_kv_heads):
            q, K, V, _, _ = _decoded(f, b, g)
            want = M.dense_attention(q, K, V, L, w.scale)
            _check_out(w, out[b, g * G:(g + 1) * G], want, q, K, V, np.arange(L),
                       f"{w.name} row ({b},{g})")


def test_dense_per_row_lengths():
    """Lengths per (sequence, KV head): empty, one token, page edges, a ragged tail, all."""
    _gpu()
    from tests.gpu_util import Filled, out_to_f64
    w = synth.small(synth.BLOCK128K)
    inp = synth.Inputs(w)
    f = Filled(inp)
    f.decode()
    rows = w.batch * w.n_kv_heads
    L0 = int(inp.lens.min())
    picks = [0, 1, 63, 64, 127, 128, 129, 1000, L0 - 1, L0]
    lens = np.array([picks[i % len(picks)] for i in range(rows)], dtype=np.int32)
    rl = torch.from_numpy(lens).cuda()
    out = out_to_f64(_dense(f, f.cache, rl, f.layer.max_context))
    G = w.group
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            n = int(lens[b * w.n_kv_heads + g])
            q, K, V, _, _ = _decoded(f, b, g)
            got = out[b, g * G:(g + 1) * G]
            want = M.dense_attention(q, K, V, n, w.scale)
            if n == 0:
                assert np.array_equal(got, np.zeros_like(got)), f"row ({b},{g}) length 0"
            else:
                _check_out(w, got, want, q, K, V, np.arange(n), f"row ({b},{g}) length {n}")


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_gather_then_attend(w):
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import GatheredKV
    from tests.gpu_util import Filled, out_to_f64
    inp = synth.Inputs(w)
    f = Filled(inp)
    out, sel, nsel = f.decode()
    gk = GatheredKV.allocate(f.layer, fill=float("nan"))
    qs.qs_gather_kv(f.cfg, f.cache, sel, nsel, w.batch, gk.k, gk.v, gk.row_lens, f.layer.ws)
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    P = gk.pages_per_seq
    d = w.head_dim
    kd = gk.k.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.batch, P, w.n_kv_heads, 128, d)
    vd = gk.v.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.batch, P, w.n_kv_heads, 128, d)
    row_lens = gk.row_lens.cpu().numpy()
    sel_h, nsel_h = sel.cpu().numpy(), nsel.cpu().numpy()
    # bits of the fill pattern, which every slot past a row's gathered length keeps
    k_nan = int(torch.full((1,), float("nan"), dtype=gk.k.dtype).view(torch.int16).item()) & 0xffff
    v_nan = int(torch.full((1,), float("nan"), dtype=gk.v.dtype).view(torch.int16).item()) & 0xffff
    for b in range(w.batch):
        L = int(inp.lens[b])
        for g in range(w.n_kv_heads):
            got_sel = sel_h[b, g, :nsel_h[b, g]]
            src, n = M.gather_blocks(got_sel, w.block_size, L)
            assert row_lens[b * w.n_kv_heads + g] == n, f"row ({b},{g}) length"
            _, _, _, kb, vb = _decoded(f, b, g)
            krow = kd[b, :, g].reshape(P * 128, d)
            vrow = vd[b, :, g].reshape(P * 128, d)
            assert np.array_equal(krow[:n], kb[src[:n]]), f"row ({b},{g}) K"
            assert np.array_equal(vrow[:n], vb[src[:n]]), f"row ({b},{g}) V"
            assert np.all(krow[n:] == k_nan) and np.all(vrow[n:] == v_nan), \
                f"row ({b},{g}) wrote past its gathered length"
    # dense attention over the compact buffer is the sparse attention over the selection
    out_g = out_to_f64(_dense(f, gk.cache(), gk.row_lens, gk.max_context))
    out_s = out_to_f64(out)
    G = w.group
    gq = query_scale_all(inp, Q=f.Q) if w.proxy_dtype == "nvfp4" else None
    for b in range(w.batch):
        L = int(inp.lens[b])
        for g in range(w.n_kv_heads):
            got_sel = sel_h[b, g, :nsel_h[b, g]]
            row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
            r = oracle_row(inp, b, g, row=row, g_q=gq, sel_override=got_sel)
            where = f"{w.name} row ({b},{g})"
            q, K, V, _, _ = _decoded(f, b, g)
            for got, how in ((out_g, " gather-then-attend"), (out_s, " gather-free")):
                _check_out(w, got[b, g * G:(g + 1) * G], r["out"], q, K, V, r["tokens"],
                           where + how)


def test_gather_reports_bad_selection_and_stays_usable():
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    from score_then_select_b200.layer import GatheredKV
    from tests.gpu_util import Filled
    w = synth.small(synth.BLOCK128K)
    inp = synth.Inputs(w)
    f = Filled(inp)
    _, sel, nsel = f.decode()
    gk = GatheredKV.allocate(f.layer)
    bad = sel.clone()
    bad[1, 3, 2] = 1 << 20                         # past the row's blocks
    qs.qs_gather_kv(f.cfg, f.cache, bad, nsel, w.batch, gk.k, gk.v, gk.row_lens, f.layer.ws)
    st = f.status()
    assert st == (B.QS_ERR_DEVICE_BOUNDS, 8, 1 * w.n_kv_heads + 3), st
    qs.qs_gather_kv(f.cfg, f.cache, sel, nsel, w.batch, gk.k, gk.v, gk.row_lens, f.layer.ws)
    assert f.status()[0] == 0


def test_dense_reports_row_longer_than_cache():
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    from score_then_select_b200.layer import workspace
    from tests.gpu_util import Filled
    w = synth.small(synth.BLOCK128K)
    inp = synth.Inputs(w)
    f = Filled(inp)
    f.decode()
    mc = f.layer.max_context
    ws = workspace(qs.qs_dense_workspace_size(f.cfg, w.batch, mc))
    rl = torch.full((w.batch * w.n_kv_heads,), 100, dtype=torch.int32, device="cuda")
    rl[5] = (-(-mc // 128) + 1) * 128               # one page more than the plan holds
    out = _out_tensor(w)
    qs.qs_dense_attn(f.cfg, f.cache, f.q, rl, w.batch, out, ws)
    st = qs.qs_device_status(ws)
    assert st[0] == B.QS_ERR_DEVICE_BOUNDS and st[1] == 6, st
    rl[5] = 100
    qs.qs_dense_attn(f.cfg, f.cache, f.q, rl, w.batch, out, ws)
    assert qs.qs_device_status(ws)[0] == 0
