"""The select kernel alone, through qs_select_topk, on crafted block scores: the GPU's
selection must equal the oracle's (forced blocks, then the best others with ties to the
lower index, ascending) exactly.

Rows cover the kernel shapes (up to 1,024, 4,096 and 32,768 blocks per row in one CTA, and
131,072 in a cluster of 4 CTAs) and the
cases the workloads rarely reach:
- heavy ties (few distinct values, which takes the radix passes);
- all scores equal;
- -0.0 next to +0.0;
- NaN and +-inf;
- extreme magnitudes;
- rows whose budget covers every block;
- the NVFP4 kept blocks.

Non-finite scores follow the rule stated in include/qs.h: NaN and -inf rank as -FLT_MAX,
+inf as FLT_MAX, ties to the lower index. The expected selection applies that map to
the input and then runs the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import method as M

pytestmark = pytest.mark.gpu

FMAX = np.float32(np.finfo(np.float32).max)


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _mapped(beta32):
    x = np.asarray(beta32, dtype=np.float32).astype(np.float64)
    x = np.where(np.isnan(x), -float(FMAX), x)
    return np.clip(x, -float(FMAX), float(FMAX))


def _scores(kind, rng, n):
    if kind == "normal":
        return rng.standard_normal(n).astype(np.float32)
    if kind == "ties":                      # ten distinct values
        return rng.integers(0, 10, n).astype(np.float32)
    if kind == "equal":
        return np.full(n, 3.25, dtype=np.float32)
    if kind == "signed_zero":
        x = rng.integers(-1, 2, n).astype(np.float32) * 0.0
        x[rng.random(n) < 0.5] = -0.0
        x[rng.random(n) < 0.01] = 1.0
        return x
    if kind == "nonfinite":
        x = rng.standard_normal(n).astype(np.float32)
        r = rng.random(n)
        x[r < 0.02] = np.nan
        x[(r >= 0.02) & (r < 0.04)] = np.inf
        x[(r >= 0.04) & (r < 0.06)] = -np.inf
        x[(r >= 0.06) & (r < 0.07)] = FMAX
        x[(r >= 0.07) & (r < 0.08)] = -FMAX
        return x
    if kind == "extreme":                   # values spanning the whole float32 range
        e = rng.uniform(-120, 120, n)
        return (np.sign(rng.standard_normal(n)) * np.exp2(e)).astype(np.float32)
    if kind == "clustered":                 # nearly equal values (many in one linear bin)
        return (1.0 + rng.integers(0, 4, n) * 2.0 ** -20).astype(np.float32)
    raise ValueError(kind)


KINDS = ["normal", "ties", "equal", "signed_zero", "nonfinite", "extreme", "clustered"]
# (block size, budget, max_context, forced sink / last): 1,024 / 4,096 / 32,768 / 131,072 blocks
SHAPES = [(128, 64, 131072, True), (32, 100, 131072, False), (1, 2048, 32768, False),
          (1, 500, 32768, True), (1, 2048, 131072, False), (1, 3000, 131072, True),
          # forced blocks fill the budget: only the sink and the last block are selected
          (128, 2, 131072, True), (1, 2, 131072, True)]


def _run(shape, kind, seed):
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import workspace
    S, budget, max_ctx, forced = shape
    rng = np.random.default_rng(seed)
    batch, Hkv = 2, 3
    nb_stride = -(-max_ctx // 128) * (128 // S)
    # lengths: the full context, and one that ends inside a block
    lens = np.array([max_ctx, max_ctx - 77 * S // 2 - 1], dtype=np.int32)
    cfg = qs.make_config(n_q_heads=Hkv * 4, n_kv_heads=Hkv, head_dim=128, block_size=S,
                         budget=budget, proxy_rank=32, proxy_dtype="bf16",
                         force_sink=forced, force_last=forced)
    beta = np.stack([_scores(kind, rng, nb_stride) for _ in range(batch * Hkv)]).reshape(
        batch, Hkv, nb_stride)
    dev = torch.device("cuda")
    seq = torch.from_numpy(lens).to(dev)
    pt = torch.zeros((batch, max_ctx // 128), dtype=torch.int32, device=dev)
    k = torch.zeros((1, Hkv, 128, 128), dtype=torch.bfloat16, device=dev)
    cache = qs.make_cache(k=k, v=k, proxy=k, page_table=pt, seq_lens=seq, max_context=max_ctx)
    ws = workspace(qs.qs_workspace_size(cfg, batch, max_ctx))
    scores = torch.from_numpy(beta).to(dev)
    sel = torch.full((batch, Hkv, budget), -7, dtype=torch.int32, device=dev)
    nsel = torch.full((batch, Hkv), -7, dtype=torch.int32, device=dev)
    qs.qs_select_topk(cfg, cache, scores, batch, sel, nsel, ws)
    st = qs.qs_device_status(ws)
    assert st[0] == 0, f"device status {st}"
    sel, nsel = sel.cpu().numpy(), nsel.cpu().numpy()
    for b in range(batch):
        nb = -(-int(lens[b]) // S)
        for g in range(Hkv):
            want = M.select_blocks(_mapped(beta[b, g, :nb]), budget,
                                   M.forced_blocks(nb, forced, forced))
            n = int(nsel[b, g])
            assert n == len(want), (b, g, n, len(want))
            assert np.array_equal(sel[b, g, :n], want), \
                f"{kind} S={S} k={budget} row ({b},{g}): {np.setdiff1d(sel[b, g, :n], want)[:8]}"
            assert np.all(sel[b, g, n:] == -1)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"S{s[0]}-k{s[1]}-L{s[2]}")
@pytest.mark.parametrize("kind", KINDS)
def test_select_matches_oracle(shape, kind):
    _gpu()
    _run(shape, kind, seed=10 * SHAPES.index(shape) + KINDS.index(kind))


def test_select_budget_covers_every_block():
    _gpu()
    # 1,024 blocks per row at most with a budget of 64: a 5,000-token row has 40 blocks
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import workspace
    cfg = qs.make_config(n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=128, budget=64,
                         proxy_rank=32, proxy_dtype="bf16", force_sink=True, force_last=True)
    dev = torch.device("cuda")
    lens = torch.tensor([5000, 1], dtype=torch.int32, device=dev)
    pt = torch.zeros((2, 1024), dtype=torch.int32, device=dev)
    k = torch.zeros((1, 2, 128, 128), dtype=torch.bfloat16, device=dev)
    cache = qs.make_cache(k=k, v=k, proxy=k, page_table=pt, seq_lens=lens, max_context=131072)
    ws = workspace(qs.qs_workspace_size(cfg, 2, 131072))
    scores = torch.randn((2, 2, 1024), device=dev)
    sel = torch.full((2, 2, 64), -7, dtype=torch.int32, device=dev)
    nsel = torch.zeros((2, 2), dtype=torch.int32, device=dev)
    qs.qs_select_topk(cfg, cache, scores, 2, sel, nsel, ws)
    assert qs.qs_device_status(ws)[0] == 0
    sel = sel.cpu().numpy()
    assert nsel.cpu().numpy().tolist() == [[40, 40], [1, 1]]
    assert sel[0, 0].tolist() == list(range(40)) + [-1] * 24
    assert sel[1, 1].tolist() == [0] + [-1] * 63


def test_select_kept_blocks():
    """NVFP4 path: the two complete blocks with the largest block error are forced."""
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import workspace
    rng = np.random.default_rng(3)
    batch, Hkv, S, budget, max_ctx = 2, 2, 128, 16, 131072
    cfg = qs.make_config(n_q_heads=8, n_kv_heads=Hkv, head_dim=128, block_size=S, budget=budget,
                         proxy_rank=0, proxy_dtype="nvfp4", v_dtype="f16", v_agg_dtype="f16",
                         force_sink=True, force_last=True, n_keep_hp=2)
    dev = torch.device("cuda")
    lens = np.array([max_ctx - 5, 40000], dtype=np.int32)
    nbs = max_ctx // S
    beta = rng.integers(0, 50, (batch, Hkv, nbs)).astype(np.float32)   # ties included
    err = rng.integers(0, 30, (batch, Hkv, nbs)).astype(np.float32)    # tied errors too
    k = torch.zeros((1, Hkv, 128, 128), dtype=torch.bfloat16, device=dev)
    # make_cache keeps raw pointers: the tensors must outlive the call
    pt = torch.zeros((batch, 1024), dtype=torch.int32, device=dev)
    seq = torch.from_numpy(lens).to(dev)
    err_d = torch.from_numpy(err).to(dev)
    cache = qs.make_cache(k=k, v=k, proxy=k, page_table=pt, seq_lens=seq, max_context=max_ctx,
                          block_err=err_d)
    ws = workspace(qs.qs_workspace_size(cfg, batch, max_ctx))
    sel = torch.full((batch, Hkv, budget), -7, dtype=torch.int32, device=dev)
    nsel = torch.zeros((batch, Hkv), dtype=torch.int32, device=dev)
    qs.qs_select_topk(cfg, cache, torch.from_numpy(beta).to(dev), batch, sel, nsel, ws)
    assert qs.qs_device_status(ws)[0] == 0
    sel = sel.cpu().numpy()
    for b in range(batch):
        L = int(lens[b])
        nb = -(-L // S)
        for g in range(Hkv):
            kept = M.kept_blocks(err[b, g, :L // S].astype(np.float64), 2)
            want = M.select_blocks(beta[b, g, :nb].astype(np.float64), budget,
                                   M.forced_blocks(nb, True, True, kept))
            assert np.array_equal(sel[b, g], want), (b, g)
