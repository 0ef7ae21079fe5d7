"""The decode step captured into a CUDA graph (CapturedDecode) gives the same bits as the
eager qs_decode call: every reduction on the path has a fixed order."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [synth.small(synth.BLOCK128K), synth.small(synth.NVFP4_128K)],
                         ids=lambda w: w.name)
def test_captured_step_matches_eager(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import score_then_select_b200 as qs
    from score_then_select_b200.graph import CapturedDecode
    from tests.gpu_util import Filled
    inp = synth.Inputs(w)
    f = Filled(inp)
    lay = f.layer
    start = lay.seq_lens.clone()
    out, sel, nsel = f.decode()
    ref_out, ref_sel = out.clone(), sel.clone()
    q_d, k_d, v_d = torch.empty_like(f.q), torch.empty_like(f.k_last), torch.empty_like(f.v_last)
    cap = CapturedDecode(f.cfg, f.cache, f.P, w.batch, out, sel, nsel, lay.ws, q_d, k_d, v_d,
                         before=lambda: lay.seq_lens.copy_(start, non_blocking=True))
    cap.q_host.copy_(f.q.cpu())
    cap.k_host.copy_(f.k_last.cpu())
    cap.v_host.copy_(f.v_last.cpu())
    for _ in range(2):
        out.zero_()
        cap.step()
        assert torch.equal(cap.out_host, ref_out.cpu())
        assert torch.equal(sel, ref_sel)
    assert qs.qs_device_status(lay.ws)[0] == 0
    assert cap.h2d_bytes == (f.q.numel() + f.k_last.numel() + f.v_last.numel()) * 2
