"""Full prefill shapes compared with the CPU oracle on every row.

The oracle is the single-threaded C program, sharded over the host's cores by token
ranges (oracle.parallel; rows are independent in the layer forward).  Qwen3.6-shaped
T = 8192 runs FC2 with 256-token tiles; Nemotron-shaped T = 4096 runs both GEMMs with
256-token tiles (FC1 ReLU^2 and FC2): the widths the sampled-row prefill tests alone
would leave unchecked on most rows."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from oracle import parallel as opar
from tests import _util

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,T,tiles", [(gen.QWEN36, 8192, (128, 256)), (gen.NEMOTRON, 4096, (256, 256))])
def test_full_prefill_every_row(shape, T, tiles):
    d = _util.device_layer(shape, T, seed=12)
    layer = moe.MoELayer(shape, _util.weights_of(d))
    desc = layer.desc(T)
    assert moe.select_path(desc) == "large"
    assert moe.token_tiles(desc) == tiles
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    got = {"out": gen.bf16_bits(out), "w": tw.cpu().numpy(), "ids": ti.cpu().numpy(), "lg": lg.cpu().numpy()}
    h = _util.host_copy(d)
    del d, layer, out, tw, ti, lg
    torch.cuda.empty_cache()
    h["router_logits"] = None
    ref_out, ref_lg, ref_w, ref_ids = opar.forward_parallel(shape, h)
    _util.check_fused_routing(got["ids"], got["w"], got["lg"], ref_ids, ref_w, ref_lg, shape, h["bias"], False)
    _util.assert_out_close(got["out"], ref_out, f"{shape.name} T={T} every row")
