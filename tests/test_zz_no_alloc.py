"""qs_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.

Such callers (a plugin of a framework that owns all device memory and passes only inputs
and outputs, or a decode loop where cudaMalloc would synchronise the device) get the same
attention with its scratch in the library's static device array instead of a workspace.
Checked through the C ABI against qs_sparse_attn on the same inputs, on two calls in a
row (the second call reuses the array the first one left behind). This file is collected
last so that a run stopping at its first failure has run every other test already.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("w", [synth.small(synth.BLOCK128K), synth.small(synth.RAGGED)],
                         ids=lambda w: w.name)
def test_noalloc_matches_workspace_attention_twice(w):
    _need_gpu()
    import score_then_select_b200 as qs
    from tests.gpu_util import Filled, out_to_f64
    f = Filled(synth.Inputs(w))
    out_ws, sel, nsel = f.decode()                       # selection + workspace attention
    out_ref = torch.zeros_like(out_ws)
    qs.qs_sparse_attn(f.cfg, f.cache, f.q, sel, nsel, w.batch, out_ref, f.layer.ws)
    torch.cuda.synchronize()
    assert qs.qs_device_status(f.layer.ws)[0] == 0
    ref = out_to_f64(out_ref)
    for call in range(2):
        out = torch.full_like(out_ref, float("nan"))
        qs.qs_sparse_attn_noalloc(f.cfg, f.cache, f.q, sel, nsel, w.batch, out)
        torch.cuda.synchronize()
        got = out_to_f64(out)
        err = np.abs(got - ref).max()
        assert err <= 2e-2, f"call {call}: max-abs {err}"


def test_noalloc_rejects_requests_beyond_its_scratch():
    _need_gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    from tests.gpu_util import Filled
    w = synth.small(synth.BLOCK128K)
    f = Filled(synth.Inputs(w))
    out = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((w.batch, w.n_kv_heads, w.budget), dtype=torch.int32, device="cuda")
    nsel = torch.zeros((w.batch, w.n_kv_heads), dtype=torch.int32, device="cuda")
    with pytest.raises(qs.QsError) as e:                 # 1024 sequences need far more
        qs.qs_sparse_attn_noalloc(f.cfg, f.cache, f.q, sel, nsel, 1024, out)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
