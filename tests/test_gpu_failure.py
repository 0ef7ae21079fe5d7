"""Failure detection on the GPU without a fault: a bounded wait that nothing can satisfy ends
with QS_ERR_DEVICE_TIMEOUT in the workspace status word, and the context stays usable."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_lost_arrival_times_out_and_is_reported():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    from tests.gpu_util import Filled, out_to_f64
    from tests.util import oracle_row
    w = synth.TINY
    inp = synth.Inputs(w)
    f = Filled(inp)
    ws = f.layer.ws
    assert f.status()[0] == 0
    qs.qs_selftest_wait_timeout(ws)
    st, kid, info = qs.qs_device_status(ws)
    assert st == B.QS_ERR_DEVICE_TIMEOUT and kid == 7
    assert qs.qs_device_status(ws)[0] == 0                 # reading it cleared it
    # the context still runs the decode step, with the oracle's result
    out, sel, nsel = f.decode()
    assert f.status()[0] == 0
    n = int(nsel[0, 0])
    r = oracle_row(inp, 0, 0, row=inp.row(0, 0), sel_override=sel[0, 0, :n].cpu().numpy())
    got = out_to_f64(out)[0, :w.group]
    rel = np.linalg.norm(got - r["out"]) / np.linalg.norm(r["out"])
    assert rel <= 1e-3
