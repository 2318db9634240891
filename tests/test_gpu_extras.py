"""The layer's optional parts on the GPU against the CPU oracle, every row, both paths:
a routed scale (the configured routed scaling factor applied to the routed output after
the router, "Laguna exact M=8 BF16-input router top-k preregistration", "Question and
arithmetic contract"), a sigmoid gate on the shared expert (the (1, H) shared-expert
gate of vLLM PR #64636's decode table), and a caller-computed shared output added in
the routed-BF16-then-shared-add order, written to a separate buffer or in place over
the shared output ("MTP1 isolated gather/shared-add closure": separate-output and
shared-output-alias forms)."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from mixture_experts_layer_35_b200.inputs import LayerShape
from tests import _util

pytestmark = pytest.mark.gpu

GATED = LayerShape("gated-H256-I192-E16-top4-swiglu-sigmoid-shared", 256, 192, 16, 4, "swiglu", "sigmoid", True,
                   0.5, 64)
GATED_R2 = LayerShape("gated-H320-I136-E8-top2-relu2-softmax-shared", 320, 136, 8, 2, "relu2", "softmax", True,
                      None, 128)
NO_SHARED = LayerShape("plain-H320-I136-E8-top2-relu2-softmax", 320, 136, 8, 2, "relu2", "softmax", True, None, 0)
NO_SHARED_SW = LayerShape("plain-H512-I256-E64-top6-swiglu-softmax", 512, 256, 64, 6, "swiglu", "softmax", True,
                          None, 0)


def _compare(shape, d, out, tw, ti, lg, scale, what):
    h = _util.host_copy(d)
    h["router_logits"] = None
    ref_out, ref_lg, ref_w, ref_ids = oracle.forward(shape, h, routed_scale=scale)
    _util.check_fused_routing(ti.cpu().numpy(), tw.cpu().numpy(), lg.cpu().numpy(), ref_ids, ref_w, ref_lg, shape,
                              h["bias"], False)
    _util.assert_out_close(gen.bf16_bits(out), ref_out, what)


@pytest.mark.parametrize("path", ["small", "large"])
@pytest.mark.parametrize("shape,T", [(GATED, 5), (GATED, 16), (GATED_R2, 3), (gen.TINY, 4)])
def test_gate_and_scale_few_tokens(shape, T, path):
    d = _util.device_layer(shape, T, seed=50 + T, shared_gate=True)
    layer = moe.MoELayer(shape, _util.weights_of(d), path=path, routed_scale=2.5)
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    _compare(shape, d, out, tw, ti, lg, 2.5, f"{shape.name} T={T} {path} gate+scale")


@pytest.mark.parametrize("shape,T", [(GATED, 300), (GATED_R2, 517), (gen.LARGE_E, 300), (gen.TINY, 100)])
def test_gate_and_scale_many_tokens(shape, T):
    """Many tokens: the gate comes from the one-kernel top-k, or (Large-E-shaped, 512
    experts) from the final kernel of the split top-k; the gated shared output from the
    FC2 epilogue; the scale from the finalize kernel."""
    d = _util.device_layer(shape, T, seed=60, shared_gate=True)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large", routed_scale=0.75)
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    if T > 200:  # the oracle on a row sample (full shapes are slow on one core)
        h = _util.host_copy(d)
        rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(T).choice(T, 24, replace=False)]))
        ref_out = oracle.forward(shape, h, rows.astype(np.int32), routed_scale=0.75)[0]
        _util.assert_out_close(gen.bf16_bits(out)[rows], ref_out, f"{shape.name} T={T} gate+scale")
        ref_lg = oracle.router_logits(h["x"], h["router_w"])
        rw, rids, _ = oracle.topk(ref_lg, shape.K, shape.score, h["bias"], shape.renorm)
        _util.check_fused_routing(ti.cpu().numpy(), tw.cpu().numpy(), lg.cpu().numpy(), rids, rw, ref_lg, shape,
                                  h["bias"], False)
    else:
        _compare(shape, d, out, tw, ti, lg, 0.75, f"{shape.name} T={T} gate+scale")


@pytest.mark.parametrize("in_place", [False, True])
@pytest.mark.parametrize("shape,T,path", [(NO_SHARED, 4, "small"), (NO_SHARED, 4, "large"), (NO_SHARED, 300, "large"),
                                          (NO_SHARED_SW, 16, "small"), (NO_SHARED_SW, 200, "large")])
def test_caller_shared_output(shape, T, path, in_place):
    d = _util.device_layer(shape, T, seed=70 + T, shared_out=True)
    layer = moe.MoELayer(shape, _util.weights_of(d), path=path, routed_scale=1.5)
    sh = d["shared_out"]
    sh_before = sh.clone()
    out = sh if in_place else torch.empty_like(sh)
    _, tw, ti, lg = layer.forward(d["x"], out=out, return_routing=True, shared_out=sh)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    if not in_place:
        assert torch.equal(sh.view(torch.int16), sh_before.view(torch.int16)), "shared_out must be read only"
    d_ref = dict(d, shared_out=sh_before)
    _compare(shape, d_ref, out, tw, ti, lg, 1.5, f"{shape.name} T={T} {path} caller shared in_place={in_place}")


def test_partially_overlapping_output_is_rejected():
    shape, T = NO_SHARED, 8
    d = _util.device_layer(shape, T, seed=3, shared_out=True)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    big = torch.empty((T + 1, shape.H), dtype=torch.bfloat16, device="cuda")
    big[:T].copy_(d["shared_out"])
    with pytest.raises(moe.MoEError) as e:
        layer.forward(d["x"], out=big[1:], shared_out=big[:T])
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError):
        layer.forward(d["x"], out=d["x"])
