"""qs_select_topk_radix (top-k by histogram passes) against qs_select_topk and the oracle,
on the crafted block scores of the select tests.

The bar: the radix selection equals qs_select_topk's exactly, and both equal the oracle's
(forced blocks, then the best others with ties to the lower index, ascending; NaN and
-inf rank as -FLT_MAX, +inf as FLT_MAX, -0 with +0), for every score kind and shape,
including rows whose budget covers every block and rows the forced blocks fill.
"""
import numpy as np
import pytest
import torch

from oracle import method as M
from tests.test_gpu_select import KINDS, SHAPES, _mapped, _scores

pytestmark = pytest.mark.gpu


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"S{s[0]}-k{s[1]}-L{s[2]}")
@pytest.mark.parametrize("kind", KINDS)
def test_radix_equals_pairwise_and_oracle(shape, kind):
    _gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import workspace
    S, budget, max_ctx, forced = shape
    rng = np.random.default_rng(100 * SHAPES.index(shape) + KINDS.index(kind))
    batch, Hkv = 2, 3
    nb_stride = -(-max_ctx // 128) * (128 // S)
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
    outs = []
    for call in (qs.qs_select_topk, qs.qs_select_topk_radix):
        sel = torch.full((batch, Hkv, budget), -7, dtype=torch.int32, device=dev)
        nsel = torch.full((batch, Hkv), -7, dtype=torch.int32, device=dev)
        call(cfg, cache, scores, batch, sel, nsel, ws)
        st = qs.qs_device_status(ws)
        assert st[0] == 0, f"device status {st}"
        outs.append((sel.cpu().numpy(), nsel.cpu().numpy()))
    (s1, n1), (s2, n2) = outs
    assert np.array_equal(n1, n2) and np.array_equal(s1, s2)
    for b in range(batch):
        nb = -(-int(lens[b]) // S)
        for g in range(Hkv):
            want = M.select_blocks(_mapped(beta[b, g, :nb]), budget,
                                   M.forced_blocks(nb, forced, forced))
            assert np.array_equal(s2[b, g, :n2[b, g]], want), (kind, shape, b, g)
