"""qs_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.

Such callers (a plugin of a framework that owns all device memory and passes only inputs
and outputs, or a decode loop where cudaMalloc would synchronise the device) get the same
attention with its scratch in the library's static device array instead of a workspace.
Checked through the C ABI against qs_sparse_attn on the same inputs, on two calls in a
row (the second call reuses the array the first one left behind). Both run the same
kernel with the same plan and a fixed merge order, so the outputs must be bit-equal.
This file is collected last so that a run stopping at its first failure has run every
other test already.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _twice_bit_equal(f, sel, nsel, batch):
    """qs_sparse_attn on the workspace, then qs_sparse_attn_noalloc twice; all bit-equal."""
    import score_then_select_b200 as qs
    w = f.w
    dt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    out_ref = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=dt,
                         device="cuda")
    qs.qs_sparse_attn(f.cfg, f.cache, f.q, sel, nsel, batch, out_ref, f.layer.ws)
    torch.cuda.synchronize()
    assert qs.qs_device_status(f.layer.ws)[0] == 0
    assert torch.isfinite(out_ref[:batch].float()).all()
    for call in range(2):
        out = torch.full_like(out_ref, float("nan"))
        qs.qs_sparse_attn_noalloc(f.cfg, f.cache, f.q, sel, nsel, batch, out)
        torch.cuda.synchronize()
        assert torch.equal(out[:batch], out_ref[:batch]), f"call {call}: outputs differ"


@pytest.mark.parametrize("w", [synth.small(synth.BLOCK128K), synth.small(synth.RAGGED)],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("attn_path", [1, 2])
def test_noalloc_matches_workspace_attention_twice(w, attn_path):
    """Both attention kernels (1: tile pipeline, 2: gather kernel)."""
    _need_gpu()
    from tests.gpu_util import Filled
    f = Filled(synth.Inputs(w), attn_path=attn_path)
    _, sel, nsel = f.decode()                            # selection through the workspace path
    _twice_bit_equal(f, sel, nsel, w.batch)


def test_noalloc_nearly_full_scratch():
    """The largest batch of the small block workload whose partials and counters still fit
    the static array: accepted, bit-equal to the workspace call twice, while one more
    sequence is rejected. Larger batches are only ever rejected on the host, before any
    launch, and every buffer is sized for the largest batch tried."""
    _need_gpu()
    import score_then_select_b200 as qs
    from score_then_select_b200 import binding as B
    from tests.gpu_util import Filled
    w = synth.small(synth.BLOCK128K).replace(batch=96)
    f = Filled(synth.Inputs(w), attn_path=1)
    _, sel, nsel = f.decode()
    out = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    fit = None
    for n in range(w.batch, 0, -1):
        try:
            qs.qs_sparse_attn_noalloc(f.cfg, f.cache, f.q, sel, nsel, n, out)
        except qs.QsError as e:
            assert e.status == B.QS_ERR_UNSUPPORTED
            continue
        fit = n
        break
    torch.cuda.synchronize()
    assert fit is not None and fit < w.batch, "the search must start above the limit"
    _twice_bit_equal(f, sel, nsel, fit)


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
