"""More parity cases of the binary proxy with a top-p budget ("RaBitQCache", Abstract),
beyond those of tests/test_gpu_rabitq.py:
- two more configurations, through the same checks: S = 32 (one 32-lane reduction per
  block), and S = 4 with d = 64 and a group of 8 query heads;
- the step call qs_decode_top_p against the four stage calls, bit for bit.
"""
import numpy as np
import pytest
import torch

from tests.test_gpu_rabitq import Case, _gpu, _ids, _t16
from tests.test_gpu_rabitq import test_block_log_masses as _log_masses
from tests.test_gpu_rabitq import test_chain_selects_valid_sets_and_attends_exactly as _chain
from tests.test_gpu_rabitq import test_writer_codes_bit_exact as _writer

pytestmark = pytest.mark.gpu

MORE = [  # (d, S, G, Hkv, budget, lens)
    (128, 32, 2, 2, 16, [1100, 257, 640]),
    (64, 4, 8, 1, 64, [513, 1024]),
]


@pytest.mark.parametrize("case", MORE, ids=_ids)
def test_writer_codes_bit_exact_more(case):
    _writer(case)


@pytest.mark.parametrize("case", MORE, ids=_ids)
def test_block_log_masses_more(case):
    _log_masses(case)


@pytest.mark.parametrize("case", MORE, ids=_ids)
def test_chain_more(case):
    _chain(case)


def test_step_call_equals_the_four_calls():
    """qs_decode_top_p (append, score, top-p, attention in one call) gives exactly what the
    four entry points give in sequence: the same kernels in the same order."""
    _gpu()
    import score_then_select_b200 as qs
    d, S, G, Hkv, budget, lens = (128, 16, 4, 2, 24, [1000, 2048, 77])
    c = Case(29, d, S, G, Hkv, budget, lens)
    B = c.batch
    b_idx = np.arange(B)
    k_last = _t16(c.K[b_idx, :, c.lens - 1]).cuda()                  # [b][Hkv][d]
    v_last = _t16(c.V[b_idx, :, c.lens - 1]).cuda()
    before = torch.from_numpy((c.lens - 1).astype(np.int32)).cuda()
    outs = []
    for fused in (False, True):
        c.layer.seq_lens.copy_(before)       # the last token is appended again, same slot
        out = torch.zeros((B, Hkv * G, d), dtype=torch.bfloat16, device="cuda")
        sel = torch.full((B, Hkv, budget), -7, dtype=torch.int32, device="cuda")
        nsel = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
        if fused:
            qs.qs_decode_top_p(c.cfg, c.cache, c.q_dev, k_last, v_last, c.R_dev, c.u_dev, 0.9,
                               B, out, sel, nsel, c.layer.ws)
        else:
            bs = torch.empty((B, Hkv, c.layer.nb_stride), dtype=torch.float32, device="cuda")
            ones = torch.ones((B,), dtype=torch.int32, device="cuda")
            qs.qs_append_kv(c.cfg, c.cache, k_last, v_last, ones, 1, c.R_dev, B, c.layer.ws)
            qs.qs_rabitq_score(c.cfg, c.cache, c.q_dev, c.R_dev, c.u_dev, B, bs, c.layer.ws)
            qs.qs_select_top_p(c.cfg, c.cache, bs, 0.9, B, sel, nsel, c.layer.ws)
            qs.qs_sparse_attn(c.cfg, c.cache, c.q_dev, sel, nsel, B, out, c.layer.ws)
        torch.cuda.synchronize()
        assert c.status()[0] == 0, c.status()
        assert c.layer.seq_lens.cpu().numpy().tolist() == list(lens)
        outs.append((out, sel, nsel))
    (o1, s1, n1), (o2, s2, n2) = outs
    assert torch.equal(s1, s2) and torch.equal(n1, n2) and torch.equal(o1, o2)


@pytest.mark.slow
def test_fullsize_binary_step_every_row():
    """The 128K token-level binary workload through qs_decode_top_p on the full batch (the
    bench's launch configuration). Every row, recomputed by the oracle in a host thread
    pool: the stored codes and factors bit-exact, 1 <= n_sel <= budget, strictly ascending
    and padded with -1, the selection a valid top-p set under the oracle's masses (band
    1e-4), and the output within max-abs 2e-2 of the oracle's attention over it and within
    the derived per-row L2 bound of tests/util.py."""
    _gpu()
    import synth
    import score_then_select_b200 as qs
    from oracle import method as M
    from tests.gpu_util import Filled, out_to_f64
    from tests.util import attention_error, decoded_row, each_row, oracle_row, top_p_params
    w = synth.RABITQ_TOKEN128K
    inp = synth.Inputs(w)
    f = Filled(inp)
    B, Hkv, G = w.batch, w.n_kv_heads, w.group
    out = torch.zeros((B, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((B, Hkv, w.budget), -7, dtype=torch.int32, device="cuda")
    nsel = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    u = torch.from_numpy(inp.u).cuda()
    qs.qs_decode_top_p(f.cfg, f.cache, f.q, f.k_last, f.v_last, f.P, u, w.top_p, B, out, sel,
                       nsel, f.layer.ws)
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    out, sel, nsel = out_to_f64(out), sel.cpu().numpy(), nsel.cpu().numpy()
    proxy = f.layer.proxy.cpu().numpy()
    p = top_p_params(w)
    d = w.head_dim

    def check(b, g):
        L = int(inp.lens[b])
        n = int(nsel[b, g])
        got = sel[b, g, :n].astype(np.int64)
        if not (1 <= n <= w.budget and np.all(np.diff(got) > 0) and got[-1] < L
                and np.all(sel[b, g, n:] == -1)):
            return "n_sel, order or padding"
        row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
        r = oracle_row(inp, b, g, row=row, sel_override=got)
        # the stored codes of the row, page by page
        npg = -(-L // 128)
        raw = proxy[inp.page_table[b, :npg].astype(np.int64), g]
        bits = raw[:, :128 * d // 8].reshape(npg * 128, d // 8)[:L]
        gk = np.ascontiguousarray(raw[:, 128 * d // 8:]).view(np.float32).reshape(-1)[:L]
        if not np.array_equal(bits, M.rabitq_pack_bits(r["bits"])):
            return "code bits differ"
        if not np.array_equal(gk.view(np.uint32), r["g"].view(np.uint32)):
            return "factors differ"
        ok, why = M.top_p_valid(r["mass"], p.p, w.budget, r["forced"], got, rel_tol=1e-4)
        if not ok:
            return f"top-p set {why}"
        q, K, V = decoded_row(w, row)
        return attention_error(w, out[b, g * G:(g + 1) * G], r["out"], q, K, V, r["tokens"])

    bad = each_row(check, [(b, g) for b in range(B) for g in range(Hkv)])
    assert not bad, f"{len(bad)} rows fail, e.g. " + "; ".join(bad[:4])
