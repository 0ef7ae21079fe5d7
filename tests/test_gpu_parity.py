"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same seeded inputs.

Sizes: the small copies of every workload (several tiles, several pages, ragged tails).
The bar:
  * writer: projected-key cache bit-exact (F32 / BF16 bits); NVFP4 codes and scales
    bit-exact;
  * block scores: float32 against float64, |diff| <= 2e-5 * max(|beta|);
  * selection: identical sets, except blocks within 1e-4 relative of the k-th score, where
    the oracle confirms the GPU's set is a valid top-k;
  * attention: max-abs <= 2e-2 (BF16 outputs), relative L2 <= 1e-3 (FP32 outputs), and
    the per-row L2 bound derived from the rounding of the softmax weights and the output
    (tests/util.py), against the oracle evaluated on the GPU's (validated) selection.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import method as M
from tests.util import check_attention, decoded_row, oracle_row, query_scale_all, row_params

pytestmark = pytest.mark.gpu

RANKR = [synth.TINY, synth.TINY_NEEDLE, synth.TINY_FP8, synth.TINY_CENTROID] + [synth.small(w) for w in
                                          (synth.TOKEN32K, synth.BLOCK128K, synth.RAGGED,
                                           synth.FP8_128K, synth.FP8_TOKEN32K,
                                           synth.CENTROID_128K, synth.CENTROID_S32)]
NVFP4 = [synth.small(synth.NVFP4_128K), synth.small(synth.NVFP4_STORE_128K)]


def _paths(ws):
    """(workload, attention kernel) cases: both kernels where the block size allows the tile
    pipeline (attn_path 1 forces it, 2 forces the gather kernel), the automatic choice
    otherwise; NVFP4 key storage is decoded by the tile pipeline only."""
    return [(w, p) for w in ws
            for p in ((1,) if w.key_storage == "nvfp4" else (1, 2) if w.block_size >= 8 else (0,))]


def _ids(case):
    w, p = case
    return f"{w.name}-path{p}"


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.gpu_util import Filled  # noqa: F401  (imports the library)


def _run_workload(w, attn_path=0):
    from tests.gpu_util import Filled, out_to_f64
    import score_then_select_b200 as qs
    inp = synth.Inputs(w)
    f = Filled(inp, attn_path=attn_path)
    out, sel, nsel = f.decode()
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    # standalone stages on the same (now complete) caches
    lay = f.layer
    scores = torch.full((w.batch, w.n_kv_heads, lay.nb_stride), np.nan, dtype=torch.float32,
                        device="cuda")
    qs.qs_score(f.cfg, f.cache, f.q, f.P, w.batch, scores, lay.ws)
    sel2 = torch.full_like(sel, -7)
    nsel2 = torch.zeros_like(nsel)
    qs.qs_select_topk(f.cfg, f.cache, scores, w.batch, sel2, nsel2, lay.ws)
    out2 = torch.zeros_like(out)
    qs.qs_sparse_attn(f.cfg, f.cache, f.q, sel2, nsel2, w.batch, out2, lay.ws)
    st = f.status()
    assert st[0] == 0, f"device status {st}"
    assert torch.equal(sel, sel2) and torch.equal(nsel, nsel2)
    assert torch.equal(out, out2)
    return inp, f, out_to_f64(out), sel.cpu().numpy(), nsel.cpu().numpy(), scores.cpu().numpy()


@pytest.mark.parametrize("case", _paths(RANKR), ids=_ids)
def test_rankr_parity(case):
    _gpu()
    w, path = case
    inp, f, out, sel, nsel, scores = _run_workload(w, path)
    G = w.group
    for b in range(w.batch):
        L = int(inp.lens[b])
        nb = -(-L // w.block_size)
        for g in range(w.n_kv_heads):
            row = inp.row(b, g)
            r = oracle_row(inp, b, g, row=row)
            where = f"{w.name} row ({b},{g})"
            # writer: bit-exact
            got_proxy = f.row_proxy(b, g)
            assert np.array_equal(got_proxy, r["cache"]), f"{where}: proxy cache differs"
            # scores
            beta = scores[b, g, :nb]
            tol = 2e-5 * max(np.abs(r["beta"]).max(), 1e-30)
            assert np.all(np.abs(beta - r["beta"]) <= tol), f"{where}: block scores"
            # selection
            n = int(nsel[b, g])
            got = sel[b, g, :n]
            assert np.all(sel[b, g, n:] == -1)
            ok, why = M.selection_valid(r["beta"], w.budget, r["forced"], got)
            assert ok, f"{where}: selection {why}"
            # attention over the GPU's selection
            rr = r if np.array_equal(got, r["sel"]) else oracle_row(inp, b, g, row=row,
                                                                     sel_override=got)
            check_attention(w, out[b, g * G:(g + 1) * G], rr["out"], row, rr["tokens"], where)


@pytest.mark.parametrize("case", _paths(NVFP4), ids=_ids)
def test_nvfp4_parity(case):
    """NVFP4 path: codes and scales bit-exact, FP4 tensor-core block scores within 1e-4 of
    the largest score, block errors within 1e-5 relative, kept blocks and selection valid
    up to near-ties, attention within the BF16 bound."""
    _gpu()
    w, path = case
    inp, f, out, sel, nsel, scores = _run_workload(w, path)
    gq = query_scale_all(inp)
    berr = f.layer.block_err.cpu().numpy()
    G = w.group
    for b in range(w.batch):
        L = int(inp.lens[b])
        nb = -(-L // w.block_size)
        for g in range(w.n_kv_heads):
            row = inp.row(b, g)
            r = oracle_row(inp, b, g, row=row, g_q=gq)
            where = f"{w.name} row ({b},{g})"
            codes, scl = f.row_proxy(b, g)
            ocodes, oscl, x32 = r["cache"]
            assert np.array_equal(scl, oscl), f"{where}: scales differ"
            assert np.array_equal(codes, ocodes), f"{where}: codes differ"
            beta = scores[b, g, :nb]
            tol = 1e-4 * max(np.abs(r["beta"]).max(), 1e-30)
            bad = np.abs(beta - r["beta"]) > tol
            assert not bad.any(), f"{where}: block scores {np.nonzero(bad)[0][:5]}"
            # block errors (float32 sums vs float64) and the kept pair they imply
            err_or = M.block_quant_error(x32, ocodes, oscl, inp.g_k, w.block_size, L)
            nfull = L // w.block_size
            eg = berr[b, g, :nfull]
            assert np.allclose(eg, err_or[:nfull], rtol=1e-5, atol=0), f"{where}: block errors"
            kept = M.kept_blocks(np.concatenate([eg.astype(np.float64), err_or[nfull:]]),
                                 w.n_keep_hp)
            okk, why = M.selection_valid(err_or[:nfull], w.n_keep_hp, np.zeros(0, np.int64), kept)
            assert okk, f"{where}: kept blocks {why}"
            forced = M.forced_blocks(nb, w.force_sink, w.force_last, kept)
            n = int(nsel[b, g])
            got = sel[b, g, :n]
            ok, why = M.selection_valid(r["beta"], w.budget, forced, got)
            assert ok, f"{where}: selection {why}"
            rr = oracle_row(inp, b, g, row=row, g_q=gq, sel_override=got, keep_override=kept)
            # with NVFP4 key storage the attended keys are the storage variant's (K_att)
            check_attention(w, out[b, g * G:(g + 1) * G], rr["out"], row, rr["tokens"], where,
                            K=rr["K_att"])


def test_needle_selected_on_gpu():
    _gpu()
    inp, f, out, sel, nsel, scores = _run_workload(synth.TINY_NEEDLE)
    assert 37 in sel[0, 0].tolist()


def test_dense_rows_reduce_to_dense_attention():
    """Ragged rows whose budget covers every block: the output is dense attention."""
    _gpu()
    w = synth.small(synth.RAGGED)
    inp, f, out, sel, nsel, scores = _run_workload(w)
    from oracle import formats as F
    for b in range(w.batch):
        L = int(inp.lens[b])
        if -(-L // w.block_size) > w.budget:
            continue
        for g in range(w.n_kv_heads):
            k, v, q = inp.row(b, g)
            dense = M.sparse_attention(F.bf16_to_f64(q), F.bf16_to_f64(k[:L]),
                                       F.bf16_to_f64(v[:L]), np.arange(L), w.scale)
            assert sel[b, g, :nsel[b, g]].tolist() == list(range(-(-L // w.block_size)))
            check_attention(w, out[b, g * w.group:(g + 1) * w.group], dense, (k, v, q),
                            np.arange(L), f"dense row {b},{g}")


@pytest.mark.parametrize("context", [16384 + 77, 40000 + 77])
def test_gather_short_selections_under_a_large_budget(context):
    """Token-level selections far shorter than the budget. The gather kernel's split plan
    covers the whole budget (every slot a sequence could select), so most splits of a row
    hold none of its tokens and must contribute nothing. At 16 K the plan's grid fits one
    wave of resident CTAs; at 40 K it does not (30 splits of 1,344 slots for 16 rows), so
    each row gets fewer CTAs than splits and a CTA takes several of its row's splits in
    turn. Rows select 0, 1, 37, 2,049, 5,000 and all of their tokens; each output matches
    the oracle's attention over the row's tokens, an empty row is 0."""
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200.filled import cfg_kwargs
    from score_then_select_b200.layer import workspace
    from tests.gpu_util import Filled, out_to_f64
    w = synth.small(synth.TOKEN32K).replace(context=context)
    inp = synth.Inputs(w)
    f = Filled(inp)
    held = inp.lens - 1                                  # tokens in the cache
    budget = int(inp.lens.max())
    cfg = qs.make_config(**dict(cfg_kwargs(w), budget=budget))
    ws = workspace(qs.qs_workspace_size(cfg, w.batch, f.layer.max_context))
    rng = np.random.default_rng(77)
    counts = [0, 1, 37, 2049, 5000, -1]                  # -1: every token
    sel = np.full((w.batch, w.n_kv_heads, budget), -1, dtype=np.int32)
    nsel = np.zeros((w.batch, w.n_kv_heads), dtype=np.int32)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            L = int(held[b])
            n = counts[(b * w.n_kv_heads + g) % len(counts)]
            n = L if n < 0 else min(n, L)
            t = np.sort(rng.choice(L, size=n, replace=False)).astype(np.int32)
            sel[b, g, :n] = t
            nsel[b, g] = n
    out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    qs.qs_sparse_attn(cfg, f.cache, f.q, torch.from_numpy(sel).cuda(),
                      torch.from_numpy(nsel).cuda(), w.batch, out, ws)
    st = qs.qs_device_status(ws)
    assert st[0] == 0, f"device status {st}"
    out = out_to_f64(out)
    G = w.group
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            n = int(nsel[b, g])
            got = out[b, g * G:(g + 1) * G]
            if n == 0:
                assert np.all(got == 0.0), f"row {b},{g}: an empty selection gives 0"
                continue
            L = int(held[b])
            row = (f.K[b, g, :L], f.V[b, g, :L], f.Q[b, g * G:(g + 1) * G])
            q, K, V = decoded_row(w, row)
            tokens = sel[b, g, :n].astype(np.int64)
            check_attention(w, got, M.sparse_attention(q, K, V, tokens, w.scale), row, tokens,
                            f"row {b},{g} ({n} tokens)")


@pytest.mark.parametrize("path", [1, 2])
def test_bad_page_table_entry_is_reported_not_faulted(path):
    """A page id outside the cache is skipped by every kernel and reported as a bounds
    error through the workspace status word (both attention kernels)."""
    _gpu()
    import score_then_select_b200 as qs
    from tests.gpu_util import Filled
    w = synth.small(synth.BLOCK128K)
    inp = synth.Inputs(w)
    f = Filled(inp, attn_path=path)
    assert f.status()[0] == 0
    f.layer.page_table[0, 3] = inp.num_pages + 5        # host-side corruption
    f.decode()
    st, kid, info = f.status()
    assert st == qs.binding.QS_ERR_DEVICE_BOUNDS
    assert f.status()[0] == 0                            # the status was cleared


def test_host_validation_rejects_before_launch():
    _gpu()
    import score_then_select_b200 as qs
    from tests.gpu_util import Filled, cfg_kwargs
    w = synth.TINY
    bad = dict(cfg_kwargs(w), head_dim=96)
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(qs.make_config(**bad), 1, 2048)
    assert e.value.status == qs.binding.QS_ERR_UNSUPPORTED
