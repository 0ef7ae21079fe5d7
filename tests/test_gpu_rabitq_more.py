"""More parity cases of the binary proxy with a top-p budget ("RaBitQCache", Abstract),
written after the first GPU run of tests/test_gpu_rabitq.py and marked gpu_pending until
they have run on a GPU (`pytest -m gpu_pending` selects them):
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

pytestmark = pytest.mark.gpu_pending

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
