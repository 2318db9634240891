"""Exact routing after the tensor-core router on activations far from N(0, 1).

With more than 64 tokens the router logits come from a tensor-core GEMM whose FP32
accumulation error is bounded per token by about 1.25 * 2^-23 * (H + 16) * |x_t|_2 *
max_e |Wr[e]|_2 (a per-instruction alignment-and-truncation model of the MMA); every
expert whose key lies within twice that bound of the K-th key is re-evaluated exactly
("Laguna exact M=8 BF16-input router top-k preregistration", "Question and arithmetic
contract": the selection is that of the exact FP32 logits).  The bound scales with the
activations, so scaled-up and outlier-heavy inputs must still route bit-exactly, and no
re-evaluated logit may fall outside its bound (the device error word stays 0).  The
Qwen3.6-shaped case runs the one-kernel top-k, the Large-E-shaped one (512 experts) the
screen / refine / final split."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from tests import _util

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("x_mode", ["scale32", "scale256", "outliers"])
@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 4096), (gen.LARGE_E, 512)])
def test_routing_exact_on_hostile_activations(shape, T, x_mode):
    d = _util.device_layer(shape, T, seed=23, x_mode=x_mode)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0, "device error word set (router bound or index check)"
    h = _util.host_copy(d)
    ref_lg = oracle.router_logits(h["x"], h["router_w"])
    rw, rids, _ = oracle.topk(ref_lg, shape.K, shape.score, h["bias"], shape.renorm)
    _util.check_fused_routing(ti.cpu().numpy(), tw.cpu().numpy(), lg.cpu().numpy(), rids, rw, ref_lg, shape,
                              h["bias"], False)
    rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(T).choice(T, 10, replace=False)]))
    ref_out = oracle.forward(shape, h, rows.astype(np.int32))[0]
    _util.assert_out_close(gen.bf16_bits(out)[rows], ref_out, f"{shape.name} T={T} x={x_mode}")
