"""Every token-tile width of the grouped tcgen05 GEMMs against the CPU oracle, on every
row, plus the fused path's internal permutation.

The many-token path picks one token-tile width per call for FC1 and one for FC2 from
the average rows per expert (FC1: 32, 64, 128 and, for ReLU^2, 256; FC2: 32, 128, 192,
256).  A mid-size layer (H 512, I 256, 8 experts, top-2) reaches each width at a token
count the oracle runs in seconds; the test asserts the width the library reports
(moe_token_tiles) and compares ids, weights and every output row with the oracle.
Skewed (Zipf) routing gives experts several tiles and ragged tails.

The fused path keeps its permutation in the workspace (moe_workspace_region): the
expert offsets must equal the oracle's byte for byte, and each expert's segment must
hold exactly the oracle's slots (the order within a segment is unspecified: slots are
placed by atomic cursors)."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from mixture_experts_layer_35_b200.inputs import LayerShape
from tests import _util

pytestmark = pytest.mark.gpu

TILE_SW = LayerShape("tiles-swiglu-H512-I256-E8-top2", 512, 256, 8, 2, "swiglu", "softmax", True, None, 0)
TILE_R2 = LayerShape("tiles-relu2-H512-I256-E8-top2", 512, 256, 8, 2, "relu2", "softmax", True, None, 0)
TILE_SH = LayerShape("tiles-swiglu-shared-H512-I256-E8-top2", 512, 256, 8, 2, "swiglu", "sigmoid", True, 0.1, 384)

CASES = [
    (TILE_SW, 20, "router", (32, 32)), (TILE_R2, 20, "router", (32, 32)),
    (TILE_SW, 150, "router", (64, 128)), (TILE_R2, 150, "router", (64, 128)),
    (TILE_SW, 300, "router", (128, 192)), (TILE_R2, 300, "router", (128, 192)),
    (TILE_SW, 800, "router", (128, 256)), (TILE_R2, 800, "router", (256, 256)),
    (TILE_SH, 800, "router", (128, 256)), (TILE_R2, 800, "zipf", (256, 256)),
    (TILE_SW, 1000, "zipf", (128, 256)), (TILE_SH, 300, "zipf", (128, 192)),
]


def check_internal_permutation(layer, desc, ws, ids_np, E):
    offsets = moe.workspace_view(desc, ws, moe.WS_OFFSETS).cpu().numpy()
    perm = moe.workspace_view(desc, ws, moe.WS_PERM).cpu().numpy()
    ref_off, ref_perm, _ = oracle.permute(ids_np, E)
    np.testing.assert_array_equal(offsets, ref_off)
    for e in range(E):
        a, b = ref_off[e], ref_off[e + 1]
        np.testing.assert_array_equal(np.sort(perm[a:b]), np.sort(ref_perm[a:b]), err_msg=f"expert {e} segment")


@pytest.mark.parametrize("shape,T,routing,tiles", CASES)
def test_every_tile_width_all_rows(shape, T, routing, tiles):
    d = _util.device_layer(shape, T, seed=T + 3, routing=routing)
    given = routing == "zipf"
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    desc = layer.desc(T, d["router_logits"])
    assert moe.token_tiles(desc) == tiles
    out, tw, ti, lg = layer.forward(d["x"], router_logits=d["router_logits"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    h = _util.host_copy(d)
    if not given:
        h["router_logits"] = None
    ref_out, ref_lg, ref_w, ref_ids = oracle.forward(shape, h)
    _util.check_fused_routing(ti.cpu().numpy(), tw.cpu().numpy(), lg.cpu().numpy(), ref_ids, ref_w, ref_lg, shape,
                              h["bias"], given)
    _util.assert_out_close(gen.bf16_bits(out), ref_out, f"{shape.name} T={T} {routing} tiles={tiles}")
    check_internal_permutation(layer, desc, layer._ws, ref_ids, shape.E)


@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 4096), (gen.LARGE_E, 256), (gen.NEMOTRON, 100)])
def test_internal_permutation_full_shapes(shape, T):
    """The fused path's offsets and per-expert slot sets at full layer shapes."""
    d = _util.device_layer(shape, T, seed=17)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    desc = layer.desc(T)
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    ids = ti.cpu().numpy()
    np.testing.assert_array_equal(moe.workspace_view(desc, layer._ws, moe.WS_TOPK_IDS).cpu().numpy().reshape(ids.shape),
                                  ids)
    check_internal_permutation(layer, desc, layer._ws, ids, shape.E)


@pytest.mark.parametrize("shape,T,tiles", [(TILE_SW, 300, (64, 256)), (TILE_R2, 300, (256, 128)),
                                           (TILE_SH, 150, (128, 32))])
def test_caller_chosen_tile_widths_all_rows(shape, T, tiles):
    """Token-tile widths forced by the caller (moe_layer_desc.fc1_tile_rows / fc2_tile_rows)
    instead of the per-call choice: every row against the oracle."""
    d = _util.device_layer(shape, T, seed=T + 5)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large", tiles=tiles)
    desc = layer.desc(T)
    assert moe.token_tiles(desc) == tiles
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    assert moe.get_error(layer._ws) == 0
    h = _util.host_copy(d)
    h["router_logits"] = None
    ref_out, ref_lg, ref_w, ref_ids = oracle.forward(shape, h)
    _util.check_fused_routing(ti.cpu().numpy(), tw.cpu().numpy(), lg.cpu().numpy(), ref_ids, ref_w, ref_lg, shape,
                              h["bias"], False)
    _util.assert_out_close(gen.bf16_bits(out), ref_out, f"{shape.name} T={T} forced tiles={tiles}")
