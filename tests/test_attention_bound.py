"""The attention output check of the GPU tests can fail: a dropped or mis-weighted block is
rejected, while the rounding the kernels do is accepted.

The check (tests/util.py, attention_error) applies the stated bars (max-abs 2e-2 on BF16
outputs, relative L2 1e-3 on FP32 outputs) and a per-row L2 bound derived from the
rounding of the softmax weights to the P.V operand format and of the output. The step it
guards is exact softmax attention over the selected original keys and values ("Joint
Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1).

All on the CPU, from the oracle: a float32 emulation of the kernels' arithmetic (64-token
chunks with a running max, weights rounded to the P format, FP32 accumulation, the output
rounded) must pass with room to spare; the oracle's output with one selected block left
out, or with one chunk's weight doubled in the log-sum-exp merge, must fail.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import method as M
from tests.util import attention_bound, attention_error, decoded_row, oracle_row, query_scale_all

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

BLOCK_SMALL = [synth.small(synth.BLOCK128K), synth.small(synth.RAGGED),
               synth.small(synth.NVFP4_128K), synth.TINY]


def _round(x, fmt):
    dt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[fmt]
    return torch.from_numpy(np.asarray(x, np.float32)).to(dt).float().numpy()


def _kernel_like(w, q, K, V, tokens, chunk=64):
    """float32 online softmax over 64-token chunks, weights rounded to the P format before
    the P.V product, output rounded to the output format."""
    q32, K32, V32 = (a.astype(np.float32) for a in (q, K[tokens], V[tokens]))
    lg = (np.float32(w.scale) * (q32 @ K32.T)).astype(np.float32)
    G = q.shape[0]
    m = np.full(G, -np.inf, np.float32)
    l = np.zeros(G, np.float32)
    o = np.zeros((G, V.shape[1]), np.float32)
    for c0 in range(0, lg.shape[1], chunk):
        x = lg[:, c0:c0 + chunk]
        mn = np.maximum(m, x.max(axis=1))
        a = np.exp(m - mn).astype(np.float32)
        p = np.exp(x - mn[:, None]).astype(np.float32)
        l = l * a + p.sum(axis=1)
        o = o * a[:, None] + _round(p, w.v_agg_dtype) @ V32[c0:c0 + chunk]
        m = mn
    return _round(o / l[:, None], w.out_dtype).astype(np.float64)


def _rows(w):
    inp = synth.Inputs(w)
    gq = query_scale_all(inp) if w.proxy_dtype == "nvfp4" else None
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            row = inp.row(b, g)
            yield b, g, row, oracle_row(inp, b, g, row=row, g_q=gq), inp, gq


@pytest.mark.parametrize("w", BLOCK_SMALL + [synth.small(synth.TOKEN32K)], ids=lambda w: w.name)
def test_kernel_rounding_passes_with_margin(w):
    for b, g, row, r, _, _ in _rows(w):
        q, K, V = decoded_row(w, row)
        got = _kernel_like(w, q, K, V, r["tokens"])
        assert attention_error(w, got, r["out"], q, K, V, r["tokens"]) is None
        bound = attention_bound(q, K, V, r["tokens"], w.scale, r["out"], w.v_agg_dtype,
                                w.out_dtype)
        assert np.linalg.norm(got - r["out"]) <= 0.5 * bound, f"row ({b},{g})"


@pytest.mark.parametrize("w", BLOCK_SMALL, ids=lambda w: w.name)
def test_every_dropped_block_is_rejected(w):
    """Leave out each selected block in turn (rows with more than one selected block): the
    oracle's output over the rest fails the check against the full selection's output."""
    n = 0
    for b, g, row, r, inp, gq in _rows(w):
        q, K, V = decoded_row(w, row)
        sel = r["sel"]
        if len(sel) < 2:
            continue
        for j in sel:
            rest = M.block_tokens(sel[sel != j], w.block_size, int(inp.lens[b]))
            got = M.sparse_attention(q, K, V, rest, w.scale)
            assert attention_error(w, got, r["out"], q, K, V, r["tokens"]) is not None, \
                f"row ({b},{g}): dropping block {j} passes"
            n += 1
    assert n >= 8


def test_heaviest_dropped_tokens_are_rejected_at_token_level():
    """Token level (S = 1): a token with little weight moves the output by less than the
    rounding does and cannot be told apart, but each row's 8 heaviest tokens can."""
    w = synth.small(synth.TOKEN32K)
    for b, g, row, r, inp, _ in _rows(w):
        q, K, V = decoded_row(w, row)
        tok = r["tokens"]
        lg = w.scale * (q @ K[tok].T)
        wgt = np.exp(lg - lg.max(axis=1, keepdims=True))
        wgt = (wgt / wgt.sum(axis=1, keepdims=True)).max(axis=0)
        for t in tok[np.argsort(-wgt)[:8]]:
            got = M.sparse_attention(q, K, V, tok[tok != t], w.scale)
            assert attention_error(w, got, r["out"], q, K, V, tok) is not None, \
                f"row ({b},{g}): dropping token {t} passes"


@pytest.mark.parametrize("w", BLOCK_SMALL[:3], ids=lambda w: w.name)
def test_misweighted_split_is_rejected(w):
    """The log-sum-exp merge of per-block partials with one block's weight doubled (its
    running max off by ln 2) fails; with every weight right it reproduces the output."""
    for b, g, row, r, inp, gq in _rows(w):
        q, K, V = decoded_row(w, row)
        L = int(inp.lens[b])
        parts = [M.attention_partial(q, K, V, M.block_tokens(np.array([j]), w.block_size, L),
                                     w.scale) for j in r["sel"]]
        ms, ls, os_ = (np.stack([p[i] for p in parts]) for i in range(3))
        ok = M.lse_combine(ms, ls, os_)
        assert attention_error(w, ok, r["out"], q, K, V, r["tokens"]) is None
        for s in (0, len(parts) // 2, len(parts) - 1):
            bad = ms.copy()
            bad[s] += np.log(2.0)
            got = M.lse_combine(bad, ls, os_)
            assert attention_error(w, got, r["out"], q, K, V, r["tokens"]) is not None, \
                f"row ({b},{g}): doubled weight of split {s} passes"


@pytest.mark.slow
def test_dropped_block_rejected_at_full_size():
    """Row (0, 0) of the 128K batch-16 workload: leaving out any one of its 64 selected
    blocks fails the check (each moves the output by several times the bound), while the
    float32 emulation of the kernels passes."""
    w = synth.BLOCK128K
    inp = synth.Inputs(w, rows=[(0, 0)])
    row = inp.row(0, 0)
    r = oracle_row(inp, 0, 0, row=row)
    q, K, V = decoded_row(w, row)
    assert attention_error(w, _kernel_like(w, q, K, V, r["tokens"]), r["out"], q, K, V,
                           r["tokens"]) is None
    sel = r["sel"]
    assert len(sel) == w.budget
    for j in sel:
        rest = M.block_tokens(sel[sel != j], w.block_size, int(inp.lens[0]))
        got = M.sparse_attention(q, K, V, rest, w.scale)
        assert attention_error(w, got, r["out"], q, K, V, r["tokens"]) is not None, \
            f"dropping block {j} passes"
