"""moe_fused_forward_noalloc through the C ABI: for callers that cannot allocate device
memory (inside CUDA-graph capture, under a fixed memory pool, or inside a host framework
that owns all allocations), the layer runs on the library's static scratch array.  Its
output must match the workspace entry point moe_fused_forward and the CPU oracle within
the layer tolerance of the other tests, on two calls in a row (the second call finds the
first call's leftovers in the shared array), and the static scratch's device error word,
read through moe_noalloc_get_error, must be clear after each call.  This file is
collected last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from tests import _util

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,T,path", [(gen.LARGE_E, 4, "small"), (gen.QWEN36, 64, "large"),
                                          (gen.TINY, 4, "large")])
def test_noalloc_matches_workspace_entry_point(shape, T, path):
    d = _util.device_layer(shape, T, seed=31)
    layer = moe.MoELayer(shape, _util.weights_of(d), path=path)
    ref, ref_w, ref_ids, _ = layer.forward(d["x"], return_routing=True)
    desc = layer.desc(T)
    assert moe.workspace_size(desc) <= moe.NOALLOC_SCRATCH_BYTES
    h = _util.host_copy(d)
    o_out, o_lg, o_w, o_ids = oracle.forward(shape, h)
    moe.noalloc_get_error()  # start from a clear error word (earlier calls in this process)
    for _ in range(2):  # two calls in a row
        out = torch.full((T, shape.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        tw = torch.empty((T, shape.K), dtype=torch.float32, device="cuda")
        ti = torch.empty((T, shape.K), dtype=torch.int32, device="cuda")
        moe.fused_forward_noalloc(desc, d["x"], out, tw, ti)
        torch.cuda.synchronize()
        assert moe.noalloc_get_error() == 0, "device error word of the static scratch is set"
        assert moe.noalloc_get_error() == 0, "a read must clear the error word"
        assert torch.equal(ti, ref_ids)
        _util.assert_w_close(tw.cpu().numpy(), ref_w.cpu().numpy())
        _util.assert_out_close(gen.bf16_bits(out), gen.bf16_bits(ref), "noalloc vs workspace entry point")
        # and against the oracle itself
        np.testing.assert_array_equal(ti.cpu().numpy(), o_ids)
        _util.assert_w_close(tw.cpu().numpy(), o_w)
        _util.assert_out_close(gen.bf16_bits(out), o_out, "noalloc vs oracle")


def test_noalloc_rejects_oversized_calls_before_launch():
    shape = gen.QWEN36
    d = _util.device_layer(shape, 1, seed=0)
    layer = moe.MoELayer(shape, _util.weights_of(d))
    desc = layer.desc(8192)  # needs ~150 MB of scratch
    assert moe.workspace_size(desc) > moe.NOALLOC_SCRATCH_BYTES
    st = moe.lib().moe_fused_forward_noalloc(ctypes.byref(desc), d["x"].data_ptr(), d["x"].data_ptr(), None, None,
                                             None, None)
    assert st == moe.MOE_ERR_WORKSPACE
