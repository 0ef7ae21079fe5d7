"""Parity of the binary proxy with a top-p budget ("RaBitQCache", Abstract) with the oracle,
through the C ABI, on seeded synthetic inputs.

Inputs: keys N(0, 1) plus a per-row offset N(0, 0.64) (so centring matters), six tokens per
row pushed 3 units along the row's query direction; queries 2 * that direction plus
N(0, 0.25) per head; V N(0, 1); one Haar rotation per KV head; the centre is the row's mean
stored key; rounding draws uniform in [0, 1). Ragged lengths with partial last pages; the
cache is filled by two appends per sequence (the writer continues a page).

The bar:
  * writer: code bits and factors g bit-exact against the oracle's float32 definition;
    K/V rows copied; seq_lens advanced;
  * block log-masses: -inf exactly where the oracle has -inf; elsewhere within a bound
    derived from float32 rounding of the estimate's five operations and of the centre's
    d-term dot product, plus the exp/log rounding;
  * top-p on crafted block scores: every GPU set valid under the oracle's float64 masses of
    the same float32 scores (relative band 1e-5), and equal to the oracle's set on the
    cases without near-ties;
  * the chain: the GPU's set valid under the oracle's own masses (band 1e-4) and the
    attention output within max-abs 2e-2 (BF16) of the oracle's attention over that set,
    and within the derived per-row L2 bound of tests/util.py.
"""
import math

import numpy as np
import pytest
import torch

from oracle import method as M
from synth.gen import to_bf16_bits
from tests.util import attention_error, attn_format

pytestmark = pytest.mark.gpu

EPS32 = 2.0 ** -24


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _t16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _haar(rng, d):
    A = rng.standard_normal((d, d))
    Q, Rq = np.linalg.qr(A)
    return (Q * np.sign(np.diag(Rq))[None, :]).astype(np.float32)


class Inputs:
    """Seeded inputs of one configuration (host arrays only)."""

    def __init__(self, seed, d, S, G, Hkv, budget, lens):
        rng = np.random.default_rng(seed)
        self.rng = rng
        self.d, self.S, self.G, self.Hkv, self.budget = d, S, G, Hkv, budget
        self.lens = np.asarray(lens, dtype=np.int64)
        B, Lmax = len(lens), int(max(lens))
        self.batch = B
        dirs = rng.standard_normal((B, Hkv, d))
        dirs /= np.linalg.norm(dirs, axis=2, keepdims=True)
        K = rng.standard_normal((B, Hkv, Lmax, d)) + 0.8 * rng.standard_normal((B, Hkv, 1, d))
        for b in range(B):
            for g in range(Hkv):
                pos = rng.choice(int(lens[b]), size=min(6, int(lens[b])), replace=False)
                K[b, g, pos] += 3.0 * dirs[b, g]
        Q = 2.0 * np.repeat(dirs, G, axis=1) + 0.5 * rng.standard_normal((B, Hkv * G, d))
        V = rng.standard_normal((B, Hkv, Lmax, d))
        self.K = to_bf16_bits(K.astype(np.float32))
        self.V = to_bf16_bits(V.astype(np.float32))
        self.Q = to_bf16_bits(Q.astype(np.float32))
        self.R = np.stack([_haar(rng, d) for _ in range(Hkv)])
        kf = (self.K.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        self.c = np.zeros((B, Hkv, d), dtype=np.float32)
        for b in range(B):
            self.c[b] = kf[b, :, :lens[b]].mean(axis=1).astype(np.float32)
        self.u = rng.random((B, Hkv, d)).astype(np.float32)

    def oracle_row(self, b, g):
        L, G = int(self.lens[b]), self.G
        bits, gk = M.rabitq_encode(self.K[b, g, :L], self.R[g], self.c[b, g])
        n, delta, vl, qbar = M.rabitq_query(self.Q[b, g * G:(g + 1) * G], self.R[g], self.u[b, g])
        s = M.rabitq_scores(bits, gk, n, delta, vl, self.c[b, g], qbar)
        return dict(bits=bits, g=gk, codes=n, delta=delta, vl=vl, qbar=qbar, s=s)


class Case(Inputs):
    """The inputs, and the layer filled through qs_append_kv."""

    def __init__(self, seed, d, S, G, Hkv, budget, lens, force=(True, True)):
        import score_then_select_b200 as qs
        from score_then_select_b200.layer import Layer
        super().__init__(seed, d, S, G, Hkv, budget, lens)
        rng, B, Lmax = self.rng, self.batch, int(max(lens))

        mpps = -(-Lmax // 128)
        num_pages = B * mpps + 3
        perm = rng.permutation(num_pages)[:B * mpps].reshape(B, mpps)
        self.page_table = perm.astype(np.int32)
        cfg_kw = dict(n_q_heads=Hkv * G, n_kv_heads=Hkv, head_dim=d, block_size=S,
                      budget=budget, proxy_rank=0, proxy_dtype="rabitq",
                      force_sink=force[0], force_last=force[1])
        self.layer = lay = Layer.allocate(cfg_kw, B, num_pages, mpps, Lmax)
        lay.page_table.copy_(torch.from_numpy(self.page_table))
        lay.key_center.copy_(torch.from_numpy(self.c))
        self.cfg, self.cache = lay.cfg, lay.cache()
        self.R_dev = torch.from_numpy(self.R).cuda()
        self.u_dev = torch.from_numpy(self.u).cuda()
        self.q_dev = _t16(self.Q).cuda()
        # two appends: the first half of each sequence, then the rest
        first = self.lens // 2
        for lo, n in ((np.zeros(B, dtype=np.int64), first), (first, self.lens - first)):
            mx = max(int(n.max()), 1)
            kn = np.zeros((B, Hkv, mx, d), dtype=np.uint16)
            vn = np.zeros((B, Hkv, mx, d), dtype=np.uint16)
            for b in range(B):
                kn[b, :, :n[b]] = self.K[b, :, lo[b]:lo[b] + n[b]]
                vn[b, :, :n[b]] = self.V[b, :, lo[b]:lo[b] + n[b]]
            qs.qs_append_kv(self.cfg, self.cache, _t16(kn).cuda(), _t16(vn).cuda(),
                            torch.from_numpy(n.astype(np.int32)).cuda(), mx, self.R_dev, B,
                            lay.ws)
        torch.cuda.synchronize()

    def status(self):
        import score_then_select_b200 as qs
        return qs.qs_device_status(self.layer.ws)

    def row_code(self, b, g):
        """The row's stored code read back in token order: packed bits [L][d/8], g [L]."""
        L, d = int(self.lens[b]), self.d
        npg = -(-L // 128)
        pages = torch.from_numpy(self.page_table[b, :npg].astype(np.int64)).cuda()
        raw = self.layer.proxy[pages, g].cpu().numpy()              # [npg][bytes per page]
        bits = raw[:, :128 * d // 8].reshape(npg * 128, d // 8)[:L]
        gk = np.ascontiguousarray(raw[:, 128 * d // 8:]).view(np.float32).reshape(-1)[:L]
        return bits, gk

CASES = [  # (d, S, G, Hkv, budget, lens)
    (128, 1, 4, 2, 256, [700, 1500, 129]),
    (128, 16, 4, 2, 24, [1000, 2048, 77]),
    (64, 128, 2, 3, 4, [900, 1280, 300]),
    (128, 64, 5, 1, 6, [1, 640, 385]),
]


def _ids(c):
    return f"d{c[0]}-S{c[1]}-G{c[2]}-kv{c[3]}-k{c[4]}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_writer_codes_bit_exact(case):
    _gpu()
    d, S, G, Hkv, budget, lens = case
    c = Case(11 + d + S, d, S, G, Hkv, budget, lens)
    assert c.status()[0] == 0, c.status()
    assert c.layer.seq_lens.cpu().numpy().tolist() == list(lens)
    for b in range(c.batch):
        L = int(lens[b])
        npg = -(-L // 128)
        pages = torch.from_numpy(c.page_table[b, :npg].astype(np.int64)).cuda()
        for g in range(Hkv):
            bits, gk = c.row_code(b, g)
            ob, og = M.rabitq_encode(c.K[b, g, :L], c.R[g], c.c[b, g])
            assert np.array_equal(bits, M.rabitq_pack_bits(ob)), (b, g)
            assert np.array_equal(gk.view(np.uint32), og.view(np.uint32)), (b, g)
            kc = c.layer.k[pages, g].reshape(npg * 128, d)[:L].view(torch.int16).cpu().numpy()
            assert np.array_equal(kc.view(np.uint16), c.K[b, g, :L])
            vc = c.layer.v[pages, g].reshape(npg * 128, d)[:L].view(torch.int16).cpu().numpy()
            assert np.array_equal(vc.view(np.uint16), c.V[b, g, :L])


def _block_lse(x, S, L):
    """log sum exp of x over each block's valid tokens (float64), -inf past the row."""
    nb = -(-L // S)
    out = np.full(nb, -np.inf)
    for j in range(nb):
        v = x[j * S:min((j + 1) * S, L)]
        m = v.max()
        out[j] = m + math.log(np.exp(v - m).sum())
    return out


def _score(c):
    import score_then_select_b200 as qs
    nbs = c.layer.nb_stride
    bs = torch.full((c.batch, c.Hkv, nbs), float("nan"), dtype=torch.float32, device="cuda")
    qs.qs_rabitq_score(c.cfg, c.cache, c.q_dev, c.R_dev, c.u_dev, c.batch, bs, c.layer.ws)
    torch.cuda.synchronize()
    return bs.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_block_log_masses(case):
    _gpu()
    d, S, G, Hkv, budget, lens = case
    c = Case(11 + d + S, d, S, G, Hkv, budget, lens)
    got = _score(c)
    assert c.status()[0] == 0, c.status()
    scale = 1.0 / math.sqrt(d)
    for b in range(c.batch):
        L = int(lens[b])
        nb, written = -(-L // S), -(-L // 128) * (128 // S)
        for g in range(Hkv):
            o = c.oracle_row(b, g)
            want = _block_lse(scale * o["s"], S, L)
            row = got[b, g]
            assert np.all(np.isneginf(row[nb:written])), (b, g)
            assert np.all(np.isfinite(row[:nb])), (b, g)
            # float32 error of g (Delta X + v_l Y) + c . qbar and of the exp / log
            mag = o["g"].astype(np.float64) * (float(o["delta"]) * 15 * d + abs(float(o["vl"])) * d)
            dot = float(np.abs(c.c[b, g].astype(np.float64) * o["qbar"]).sum())
            tol = scale * (4 * EPS32 * mag.max() + 4 * EPS32 * np.abs(o["s"]).max() +
                           d * EPS32 * dot) + 8 * EPS32 * max(1.0, np.abs(want).max())
            err = np.abs(row[:nb] - want).max()
            assert err <= tol, f"row ({b}, {g}): error {err:.3e} > {tol:.3e}"


def _oracle_top_p(scores32, p, budget, forced):
    x = scores32.astype(np.float32).astype(np.float64)
    x = np.where(np.isnan(x), -np.inf, np.minimum(x, np.finfo(np.float32).max))
    M_ = x.max() if x.size else -np.inf
    mass = np.zeros_like(x) if not np.isfinite(M_) else np.exp(x - M_)
    return mass, M.select_top_p(mass, p, budget, forced)


def _run_top_p(scores, L, S, budget, p, force):
    """qs_select_top_p on one row of crafted block scores (float32)."""
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    nb = len(scores)
    cfg = qs.make_config(n_q_heads=1, n_kv_heads=1, head_dim=128, block_size=S, budget=budget,
                         proxy_rank=0, proxy_dtype="rabitq", force_sink=force[0],
                         force_last=force[1])
    max_ctx = max(L, 1)
    nbs = -(-max_ctx // 128) * (128 // S)
    assert nb <= nbs
    ws = torch.zeros((qs.qs_workspace_size(cfg, 1, max_ctx),), dtype=torch.uint8, device="cuda")
    qs.qs_workspace_init(ws, ws.numel())
    sc = torch.full((1, 1, nbs), float("nan"), dtype=torch.float32, device="cuda")
    sc[0, 0, :nb] = torch.from_numpy(scores.astype(np.float32))
    lens = torch.tensor([L], dtype=torch.int32, device="cuda")
    cache = B.qs_cache()
    cache.seq_lens = lens.data_ptr()
    cache.max_context = max_ctx
    sel = torch.full((1, 1, budget), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((1, 1), -7, dtype=torch.int32, device="cuda")
    qs.qs_select_top_p(cfg, cache, sc, p, 1, sel, nsel, ws)
    st = qs.qs_device_status(ws)
    assert st[0] == 0, st
    n = int(nsel.item())
    s = sel[0, 0].cpu().numpy()
    assert 0 <= n <= budget and np.all(s[n:] == -1) and np.all(s[:n] >= 0)
    return s[:n].astype(np.int64)


def _crafted():
    rng = np.random.default_rng(3)
    out = []
    x = (rng.standard_normal(1000) * 3).astype(np.float32)
    for p in (0.1, 0.5, 0.9, 0.99, 1.0):
        for budget, force in ((64, (False, False)), (1000, (True, True)), (2000, (True, False))):
            out.append((f"normal-p{p}-k{budget}-f{int(force[0])}{int(force[1])}", x, 1, budget,
                        p, force))
    out.append(("integer-ties", np.round(rng.standard_normal(5000)).astype(np.float32), 1,
                4096, 0.5, (True, True)))
    out.append(("all-equal", np.full(300, 2.5, dtype=np.float32), 1, 300, 0.375, (False, False)))
    y = rng.standard_normal(100).astype(np.float32)
    y[::7] = -np.inf
    y[3::11] = np.nan
    out.append(("inf-nan", y, 1, 50, 0.8, (True, True)))
    out.append(("one-block", np.array([0.3], dtype=np.float32), 1, 2, 0.5, (True, True)))
    out.append(("all-neg-inf", np.full(10, -np.inf, dtype=np.float32), 1, 5, 0.5, (True, True)))
    out.append(("large", (rng.standard_normal(131072) * 4).astype(np.float32), 1, 4096, 0.9,
                (True, True)))
    out.append(("blocks-S16", (rng.standard_normal(200) * 2).astype(np.float32), 16, 40, 0.7,
                (True, True)))
    # budgets above 4,096 blocks take the histogram kernel instead of the sorted candidates
    out.append(("large-budget", (rng.standard_normal(20000) * 2).astype(np.float32), 1, 6000,
                0.9, (True, True)))
    out.append(("integer-ties-large-budget", np.round(rng.standard_normal(9000)).astype(np.float32),
                1, 5000, 0.6, (True, False)))
    return out


@pytest.mark.parametrize("case", _crafted(), ids=lambda c: c[0])
def test_top_p_on_crafted_scores(case):
    _gpu()
    name, scores, S, budget, p, force = case
    nb = len(scores)
    L = nb * S - (S // 2 if S > 1 else 0)              # a ragged last block when S > 1
    got = _run_top_p(scores, L, S, budget, p, force)
    forced = M.forced_blocks(nb, force[0], force[1])
    p32 = float(np.float32(p))                         # the ABI takes p as a float
    mass, want = _oracle_top_p(scores, p32, budget, forced)
    ok, why = M.top_p_valid(mass, p32, budget, forced, got, rel_tol=1e-5)
    assert ok, f"{name}: {why} (got {len(got)}, oracle {len(want)})"
    if name in ("all-equal", "one-block", "all-neg-inf", "inf-nan", "integer-ties",
                "integer-ties-large-budget"):
        assert np.array_equal(got, want), name
    if name == "all-equal":
        assert len(got) == math.ceil(0.375 * 300)     # equal masses: the lowest indices


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_chain_selects_valid_sets_and_attends_exactly(case):
    _gpu()
    import score_then_select_b200 as qs
    d, S, G, Hkv, budget, lens = case
    c = Case(11 + d + S, d, S, G, Hkv, budget, lens)
    nbs = c.layer.nb_stride
    bs = torch.empty((c.batch, Hkv, nbs), dtype=torch.float32, device="cuda")
    qs.qs_rabitq_score(c.cfg, c.cache, c.q_dev, c.R_dev, c.u_dev, c.batch, bs, c.layer.ws)
    p = 0.9
    sel = torch.full((c.batch, Hkv, budget), -7, dtype=torch.int32, device="cuda")
    nsel = torch.zeros((c.batch, Hkv), dtype=torch.int32, device="cuda")
    qs.qs_select_top_p(c.cfg, c.cache, bs, p, c.batch, sel, nsel, c.layer.ws)
    out = torch.zeros((c.batch, Hkv * G, d), dtype=torch.bfloat16, device="cuda")
    qs.qs_sparse_attn(c.cfg, c.cache, c.q_dev, sel, nsel, c.batch, out, c.layer.ws)
    torch.cuda.synchronize()
    assert c.status()[0] == 0, c.status()
    sel, nsel = sel.cpu().numpy(), nsel.cpu().numpy()
    out = out.float().cpu().numpy().astype(np.float64)
    scale = 1.0 / math.sqrt(d)
    for b in range(c.batch):
        L = int(lens[b])
        nb = -(-L // S)
        forced = M.forced_blocks(nb, True, True)
        kf = (c.K[b].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        vf = (c.V[b].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qf = (c.Q[b].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        for g in range(Hkv):
            o = c.oracle_row(b, g)
            mass = M.block_mass(M.estimated_weights(o["s"], scale), S)
            got = sel[b, g, :nsel[b, g]].astype(np.int64)
            ok, why = M.top_p_valid(mass, float(np.float32(p)), budget, forced, got,
                                    rel_tol=1e-4)
            assert ok, f"row ({b}, {g}): {why}"
            toks = M.block_tokens(got, S, L)
            qg = qf[g * G:(g + 1) * G]
            want = M.sparse_attention(qg, kf[g, :L], vf[g, :L], toks, scale)
            why = attention_error(attn_format(scale), out[b, g * G:(g + 1) * G], want, qg,
                                  kf[g, :L], vf[g, :L], toks)
            assert why is None, f"row ({b}, {g}): {why}"

