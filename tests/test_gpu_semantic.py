"""Parity of the semantic-block path ("Coarse Semantic Blocks ...", Abstract) with the
oracle, through the C ABI.

Inputs: per row, keys drawn around 6 centres N(0, 9 I) with N(0, 0.25 I) noise, so the
clusters are non-contiguous; V and q N(0, 1); ragged lengths; the index covers a prefix
(the prompt) and the rest of each sequence is decoded after it.

The bar:
  * index: every assignment, every centroid (float32 bits) and the member lists bit-exact
    against the oracle's float32 k-means (kmeans_keys_f32); members ascending within each
    cluster; offsets[C] = L0;
  * selection: the attended token set equals the oracle's (the top clusters' members and
    every token after the prompt), or differs only by clusters within the near-tie band of
    the k-th cluster score;
  * attention (token-level kernel over that set): max-abs <= 2e-2 (BF16 output) and the
    derived per-row L2 bound of tests/util.py.
"""
import math

import numpy as np
import pytest
import torch

from oracle import method as M
from synth.gen import to_bf16_bits
from tests.util import attention_error, attn_format

pytestmark = pytest.mark.gpu


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _t16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class SemCase:
    def __init__(self, seed, d, S, G, Hkv, budget, lens, prompts, iters):
        import score_then_select_b200 as qs
        from score_then_select_b200.layer import Layer
        rng = np.random.default_rng(seed)
        self.d, self.S, self.G, self.Hkv, self.budget, self.iters = d, S, G, Hkv, budget, iters
        self.lens = np.asarray(lens, dtype=np.int64)
        self.prompts = np.asarray(prompts, dtype=np.int64)
        B, Lmax = len(lens), int(max(lens))
        self.batch = B
        K = np.empty((B, Hkv, Lmax, d))
        for b in range(B):
            for g in range(Hkv):
                centres = rng.standard_normal((6, d)) * 3.0
                K[b, g] = centres[rng.integers(0, 6, size=Lmax)] + 0.5 * rng.standard_normal((Lmax, d))
        self.K = to_bf16_bits(K.astype(np.float32))
        self.V = to_bf16_bits(rng.standard_normal((B, Hkv, Lmax, d)).astype(np.float32))
        self.Q = to_bf16_bits(rng.standard_normal((B, Hkv * G, d)).astype(np.float32))
        mpps = -(-Lmax // 128)
        num_pages = B * mpps + 2
        self.page_table = rng.permutation(num_pages)[:B * mpps].reshape(B, mpps).astype(np.int32)
        self.cfg_kw = dict(n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=d, block_size=S,
                           budget=budget, proxy_rank=0, proxy_dtype="semantic")
        self.layer = lay = Layer.allocate(self.cfg_kw, B, num_pages, mpps, Lmax)
        lay.page_table.copy_(torch.from_numpy(self.page_table))
        self.cfg, self.cache = lay.cfg, lay.cache()
        first = self.lens // 2
        for lo, n in ((np.zeros(B, dtype=np.int64), first), (first, self.lens - first)):
            mx = max(int(n.max()), 1)
            kn = np.zeros((B, Hkv, mx, d), dtype=np.uint16)
            vn = np.zeros((B, Hkv, mx, d), dtype=np.uint16)
            for b in range(B):
                kn[b, :, :n[b]] = self.K[b, :, lo[b]:lo[b] + n[b]]
                vn[b, :, :n[b]] = self.V[b, :, lo[b]:lo[b] + n[b]]
            qs.qs_append_kv(self.cfg, self.cache, _t16(kn).cuda(), _t16(vn).cuda(),
                            torch.from_numpy(n.astype(np.int32)).cuda(), mx, None, B, lay.ws)
        rows = B * Hkv
        self.c_max = -(-Lmax // S)
        self.cent = torch.full((rows, self.c_max, d), float("nan"), dtype=torch.float32,
                               device="cuda")
        self.offsets = torch.full((rows, self.c_max + 1), -7, dtype=torch.int32, device="cuda")
        self.members = torch.full((rows, Lmax), -7, dtype=torch.int32, device="cuda")
        self.prompt_dev = torch.from_numpy(self.prompts.astype(np.int32)).cuda()
        nb = qs.qs_semantic_index_workspace_size(self.cfg, B, Lmax)
        self.ws_idx = torch.zeros((nb,), dtype=torch.uint8, device="cuda")
        qs.qs_workspace_init(self.ws_idx, nb)
        qs.qs_semantic_index(self.cfg, self.cache, self.prompt_dev, iters, self.cent,
                             self.offsets, self.members, B, self.ws_idx)
        torch.cuda.synchronize()
        st = qs.qs_device_status(self.ws_idx)
        assert st[0] == 0, st
        self.q_dev = _t16(self.Q).cuda()

    def oracle_index(self, b, g):
        L0 = int(self.prompts[b])
        C = -(-L0 // self.S)
        return M.kmeans_keys_f32(self.K[b, g, :L0], C, self.iters)


CASES = [  # (d, S, G, Hkv, budget, lens, prompts, iters)
    (128, 64, 4, 2, 3, [1500, 900, 2100], [1493, 900, 1970], 4),
    (64, 32, 2, 1, 8, [700, 1300], [690, 1300], 3),
    (128, 128, 8, 1, 2, [400, 1000], [0, 1000], 2),
]


def _ids(c):
    return f"d{c[0]}-S{c[1]}-G{c[2]}-kv{c[3]}-k{c[4]}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_index_bit_exact(case):
    _gpu()
    c = SemCase(41 + case[0] + case[1], *case)
    cent = c.cent.cpu().numpy()
    offs = c.offsets.cpu().numpy()
    mem = c.members.cpu().numpy()
    for b in range(c.batch):
        L0 = int(c.prompts[b])
        C = -(-L0 // c.S)
        for g in range(c.Hkv):
            row = b * c.Hkv + g
            assert offs[row, C] == L0 and offs[row, 0] == 0
            if C == 0:
                continue
            a32, c32 = c.oracle_index(b, g)
            got = np.full(L0, -1, dtype=np.int64)
            for j in range(C):
                m = mem[row, offs[row, j]:offs[row, j + 1]]
                assert np.all(np.diff(m) > 0), (row, j)
                got[m] = j
            assert np.array_equal(got, a32), (row, int((got != a32).sum()))
            assert np.array_equal(cent[row, :C].view(np.uint32), c32.view(np.uint32)), row


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_selection_and_attention(case):
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    c = SemCase(41 + case[0] + case[1], *case)
    Bn, Lmax = c.batch, int(c.lens.max())
    rows, max_tokens = Bn * c.Hkv, Lmax
    tokens = torch.full((rows, max_tokens), -7, dtype=torch.int32, device="cuda")
    n_tokens = torch.zeros((rows,), dtype=torch.int32, device="cuda")
    qs.qs_semantic_select(c.cfg, c.cache, c.q_dev, c.prompt_dev, c.cent, c.offsets, c.members,
                          Bn, tokens, n_tokens, max_tokens, c.layer.ws)
    tok_kw = dict(c.cfg_kw, block_size=1, budget=max_tokens)
    cfg_tok = B.make_config(**tok_kw)
    ws_tok = torch.zeros((qs.qs_workspace_size(cfg_tok, Bn, Lmax),), dtype=torch.uint8,
                         device="cuda")
    qs.qs_workspace_init(ws_tok, ws_tok.numel())
    out = torch.zeros((Bn, c.Hkv * c.G, c.d), dtype=torch.bfloat16, device="cuda")
    qs.qs_sparse_attn(cfg_tok, c.cache, c.q_dev, tokens.view(Bn, c.Hkv, max_tokens),
                      n_tokens.view(Bn, c.Hkv), Bn, out, ws_tok)
    torch.cuda.synchronize()
    for ws in (c.layer.ws, ws_tok):
        st = qs.qs_device_status(ws)
        assert st[0] == 0, st
    tok, ntok = tokens.cpu().numpy(), n_tokens.cpu().numpy()
    out = out.float().cpu().numpy().astype(np.float64)
    scale = 1.0 / math.sqrt(c.d)
    for b in range(Bn):
        L, L0 = int(c.lens[b]), int(c.prompts[b])
        for g in range(c.Hkv):
            row = b * c.Hkv + g
            got = tok[row, :ntok[row]].astype(np.int64)
            assert np.all(tok[row, ntok[row]:] == -1)
            assert len(np.unique(got)) == len(got)
            a32, c32 = c.oracle_index(b, g) if L0 > 0 else (np.zeros(0, np.int64), None)
            if L0 > 0:
                beta = M.semantic_block_scores(c.Q[b, g * c.G:(g + 1) * c.G],
                                               c32.astype(np.float64))
                want_sel = M.select_blocks(beta, c.budget, np.zeros(0, dtype=np.int64))
                want = M.semantic_tokens(a32, want_sel, L0, L)
                if not np.array_equal(np.sort(got), want):
                    # a near tie at the k-th cluster score: the GPU's clusters (inferred from
                    # its tokens; an empty cluster leaves no trace) must be a valid top set
                    got_sel = np.unique(a32[got[got < L0]])
                    nonempty = want_sel[np.bincount(a32, minlength=len(beta))[want_sel] > 0]
                    assert len(got_sel) == len(nonempty), f"row {row}: cluster count"
                    s_star, tau = M.kth_threshold(beta, c.budget, np.zeros(0, dtype=np.int64))
                    extra = np.setdiff1d(got_sel, want_sel)
                    missing = np.setdiff1d(nonempty, got_sel)
                    assert np.all(beta[extra] >= s_star - tau), f"row {row}: {extra}"
                    assert np.all(beta[missing] <= s_star + tau), f"row {row}: {missing}"
                    want = M.semantic_tokens(a32, got_sel, L0, L)
                    assert np.array_equal(np.sort(got), want), row
            else:
                want = np.arange(L)
                assert np.array_equal(np.sort(got), want), row
            q = _f64(c.Q[b, g * c.G:(g + 1) * c.G])
            Kd, Vd = _f64(c.K[b, g, :L]), _f64(c.V[b, g, :L])
            o = M.sparse_attention(q, Kd, Vd, want, scale)
            why = attention_error(attn_format(scale), out[b, g * c.G:(g + 1) * c.G], o, q, Kd,
                                  Vd, want)
            assert why is None, f"row {row}: {why}"
