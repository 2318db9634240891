"""The optional phase trace of the tensor-core kernels (the kind of per-phase scheduler
telemetry the Rocket GB10 note tabulates): tracing leaves the results unchanged, every
launched CTA stamps its phases in order, and the work units the CTAs report add up to
the call's tiles (whole tiles) or at least cover them (stream-K segments)."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from tests import _util

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 300), (gen.LARGE_E, 16), (gen.NEMOTRON, 1)])
def test_trace_stamps_are_ordered_and_results_unchanged(shape, T):
    d = _util.device_layer(shape, T, seed=3)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    ref, ref_w, ref_ids, _ = layer.forward(d["x"], return_routing=True)
    trace = moe.trace_buffer("cuda")
    out, tw, ti, _ = layer.forward(d["x"], return_routing=True, trace=trace)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    assert torch.equal(ti, ref_ids)
    _util.assert_w_close(tw.cpu().numpy(), ref_w.cpu().numpy())
    _util.assert_out_close(gen.bf16_bits(out), gen.bf16_bits(ref), "traced vs untraced")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    t = trace.view(3, moe.TRACE_MAX_CTAS, moe.TRACE_FIELDS).cpu().numpy()
    desc = layer.desc(T)
    fc1_rows, fc2_rows = moe.token_tiles(desc)
    for k in (1, 2):  # FC1, FC2: one CTA per SM
        r = t[k, :sms]
        assert (r[:, 0] > 0).all(), "every CTA stamps its entry"
        assert (r[:, 1] >= r[:, 0]).all() and (r[:, 4] >= r[:, 1]).all()
        assert (r[:, 3] <= r[:, 4]).all()
        busy = r[:, 5] > 0
        assert (r[busy, 2] >= r[busy, 1]).all()
        assert (t[k, sms:] == 0).all(), "rows past the grid stay untouched"
        assert r[:, 5].sum() > 0
    s = moe.trace_summary(trace, sms)
    assert "fc1" in s and "fc2" in s and s["fc1"]["kernel_us"] > 0
