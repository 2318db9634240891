"""moe_fused_forward on the GPU against the CPU oracle, through the C ABI.

Routing ids must match bit-exactly on every row and routing weights within 1e-6
relative (tests/_util.check_fused_routing); layer output within max-abs <= 1e-2 max|ref|
and mean-abs <= 1e-3 max|ref|.  Hand-derived fixtures must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from mixture_experts_layer_35_b200.inputs import LayerShape
from tests import _golden, _util

pytestmark = pytest.mark.gpu


def _run(shape, d, path, given_logits=False):
    layer = moe.MoELayer(shape, _util.weights_of(d), path=path)
    out, tw, ti, lg = layer.forward(d["x"], router_logits=d["router_logits"] if given_logits else None,
                                    return_routing=True)
    torch.cuda.synchronize()
    return out, tw, ti, lg


def _check(shape, d, path, rows=None, given_logits=False):
    out, tw, ti, lg = _run(shape, d, path, given_logits)
    h = _util.host_copy(d)
    if not given_logits:
        h["router_logits"] = None
    T = d["x"].shape[0]
    sel = np.arange(T) if rows is None else np.asarray(rows)
    ref_out, ref_lg, ref_w, ref_ids = oracle.forward(shape, h, sel.astype(np.int32))
    bias = h["bias"]
    same = _util.check_fused_routing(ti.cpu().numpy()[sel], tw.cpu().numpy()[sel], lg.cpu().numpy()[sel],
                                     ref_ids, ref_w, ref_lg, shape, bias, given_logits)
    got = gen.bf16_bits(out)[sel]
    return _util.assert_out_close(got[same], ref_out[same], f"{shape.name} T={T} path={path}")


def _fixture_device(name):
    shape, h, fx = _golden.layer_fixture(name)
    d = {}
    for k, v in h.items():
        if v is None:
            d[k] = None
        elif v.dtype == np.uint16:
            d[k] = gen.bits_to_bf16(v).cuda()
        else:
            d[k] = torch.from_numpy(v).cuda()
    return shape, d, fx


@pytest.mark.parametrize("path", ["small", "large"])
@pytest.mark.parametrize("name", ["combine_order.json", "relu2_integer.json", "h_rounding.json"])
def test_golden_fixtures_bit_exact(name, path):
    shape, d, fx = _fixture_device(name)
    out, tw, ti, lg = _run(shape, d, path, given_logits=True)
    np.testing.assert_array_equal(gen.bf16_bits(out), _golden.hex_bits(fx["expected_out_bits"]))
    if "expected_ids" in fx:
        assert ti.cpu().tolist() == fx["expected_ids"]


@pytest.mark.parametrize("path", ["small", "large"])
def test_tiny_config(path):
    d = _util.device_layer(gen.TINY, 4, seed=0)
    _check(gen.TINY, d, path)


MULTI_A = LayerShape("multi-a", 256, 192, 16, 4, "swiglu", "sigmoid", True, 0.5, 64)
MULTI_B = LayerShape("multi-b", 320, 136, 8, 2, "relu2", "softmax", True, None, 0)
MULTI_C = LayerShape("multi-c", 512, 256, 64, 6, "swiglu", "softmax", True, None, 128)


@pytest.mark.parametrize("shape,T", [(MULTI_A, 300), (MULTI_B, 517), (MULTI_C, 1000), (MULTI_A, 129),
                                     (MULTI_B, 1), (MULTI_C, 40)])
def test_multi_tile_ragged_large_path(shape, T):
    d = _util.device_layer(shape, T, seed=T)
    _check(shape, d, "large")


@pytest.mark.parametrize("shape", [MULTI_A, MULTI_B, MULTI_C])
@pytest.mark.parametrize("T", [1, 5, 16])
def test_small_path_and_path_parity(shape, T):
    d = _util.device_layer(shape, T, seed=100 + T)
    _check(shape, d, "small")
    o_s, w_s, i_s, _ = _run(shape, d, "small")
    o_l, w_l, i_l, _ = _run(shape, d, "large")
    assert torch.equal(i_s, i_l)
    _util.assert_out_close(gen.bf16_bits(o_l), gen.bf16_bits(o_s), "small vs large path")


@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 1), (gen.QWEN36, 4), (gen.QWEN36, 16), (gen.NEMOTRON, 1),
                                     (gen.NEMOTRON, 3), (gen.LARGE_E, 4), (gen.LARGE_E, 16)])
def test_full_shapes_decode_all_rows(shape, T):
    d = _util.device_layer(shape, T, seed=T)
    _check(shape, d, "auto")


@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 16), (gen.NEMOTRON, 16), (gen.LARGE_E, 16), (gen.NEMOTRON, 9),
                                     (gen.LARGE_E, 11)])
def test_full_shapes_small_path_max_tokens(shape, T):
    """The streaming path at its largest token counts, where x takes most of the shared
    memory and the stage ring is shortest."""
    d = _util.device_layer(shape, T, seed=40 + T)
    _check(shape, d, "small")
    layer = moe.MoELayer(shape, _util.weights_of(d), path="small")
    o1 = layer.forward(d["x"])
    o2 = layer.forward(d["x"])
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("shape,T,routing,nrows", [
    (gen.QWEN36, 4096, "router", 24), (gen.QWEN36, 2048, "zipf", 24), (gen.QWEN36, 8192, "router", 12),
    (gen.NEMOTRON, 1024, "router", 8), (gen.NEMOTRON, 4096, "zipf", 6), (gen.LARGE_E, 256, "router", 16),
    (gen.LARGE_E, 4096, "router", 8)])
def test_full_shapes_prefill_sampled_rows(shape, T, routing, nrows):
    d = _util.device_layer(shape, T, seed=11, routing=routing)
    rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(T).choice(T, nrows, replace=False)]))
    _check(shape, d, "auto", rows=rows, given_logits=(routing == "zipf"))


@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 4096), (gen.LARGE_E, 512), (gen.NEMOTRON, 300), (MULTI_A, 2000)])
def test_fused_routing_every_row(shape, T):
    """Tensor-core router + FP64 refine: ids bit-exact and weights within 1e-6 on every
    row of the batch, against the oracle's logits and top-k over all rows."""
    d = _util.device_layer(shape, T, seed=21)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    out, tw, ti, lg = layer.forward(d["x"], return_routing=True)
    torch.cuda.synchronize()
    h = _util.host_copy(d)
    ref_lg = oracle.router_logits(h["x"], h["router_w"])
    rw, rids, _ = oracle.topk(ref_lg, shape.K, shape.score, h["bias"], shape.renorm)
    _util.check_fused_routing(ti.cpu().numpy(), tw.cpu().numpy(), lg.cpu().numpy(), rids, rw, ref_lg, shape,
                              h["bias"], False)


TIED = LayerShape("tied-router", 256, 128, 320, 4, "swiglu", "softmax", True, None, 0)


@pytest.mark.parametrize("T", [100, 300])
def test_many_candidates_fall_back_to_per_row_refinement(T):
    """Every expert has the same router row, so all 320 logits of a row tie and every expert
    is a top-k candidate (more than the 32 the three-kernel top-k carries per row): those
    rows take the per-row refinement path, and the lower-id tie break must hold exactly."""
    d = _util.device_layer(TIED, T, seed=5)
    d["router_w"] = d["router_w"][:1].expand_as(d["router_w"]).contiguous()
    _check(TIED, d, "large")


@pytest.mark.parametrize("T", [16, 64])
def test_tied_router_few_tokens(T):
    """Few tokens on the many-token path (exact few-token router, top-k, permute).  Every
    expert has the same router row, so all logits of a row tie and the lower-id tie break
    decides every slot."""
    d = _util.device_layer(TIED, T, seed=6)
    d["router_w"] = d["router_w"][:1].expand_as(d["router_w"]).contiguous()
    _check(TIED, d, "large")


@pytest.mark.parametrize("shape,T", [(MULTI_A, 37), (MULTI_C, 3), (gen.LARGE_E, 64)])
def test_given_logits_few_tokens(shape, T):
    """Caller-supplied logits at few tokens on the many-token path, skewed routing so that
    some experts take many slots and most take none."""
    d = _util.device_layer(shape, T, seed=8, routing="zipf")
    _check(shape, d, "large", given_logits=True)


def test_small_path_deterministic_and_graph_replay():
    shape = gen.QWEN36
    d = _util.device_layer(shape, 4, seed=5)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="small")
    o1 = layer.forward(d["x"])
    o2 = layer.forward(d["x"])
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    out = torch.empty_like(o1)
    layer.forward(d["x"], out=out)  # warm-up outside capture (workspace allocation)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        layer.forward(d["x"], out=out, stream=s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), o1.view(torch.int16))


def test_large_path_graph_replay():
    shape = MULTI_A
    d = _util.device_layer(shape, 300, seed=9)
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large")
    ref = layer.forward(d["x"])
    out = torch.empty_like(ref)
    layer.forward(d["x"], out=out)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        layer.forward(d["x"], out=out, stream=s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    _util.assert_out_close(gen.bf16_bits(out), gen.bf16_bits(ref), "graph replay")


def test_zero_tokens():
    shape = gen.TINY
    d = _util.device_layer(shape, 1, seed=0)
    layer = moe.MoELayer(shape, _util.weights_of(d))
    x = torch.empty((0, shape.H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, shape.H), dtype=torch.bfloat16, device="cuda")
    desc = layer.desc(0)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    moe.fused_forward_raw(desc, x, out, ws)
