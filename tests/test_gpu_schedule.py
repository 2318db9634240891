"""The dynamic tile schedule of the grouped GEMMs (moe_layer_desc.schedule) against the CPU
oracle: every token-tile width on every row, and full layer shapes on sampled rows, with
the phase trace showing that the CTAs' tiles add up to the call's tiles.

With the dynamic schedule each CTA takes its next tile from a device counter, so which
CTA computes a tile changes from run to run; the results may differ from the static
schedule's only in the FP32 order of the routed combine, which is unspecified anyway."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen
from tests import _util
from tests.test_gpu_tiles import CASES, check_internal_permutation

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,T,routing,tiles", CASES)
def test_dynamic_schedule_every_tile_width_all_rows(shape, T, routing, tiles):
    d = _util.device_layer(shape, T, seed=T + 11, routing=routing)
    given = routing == "zipf"
    layer = moe.MoELayer(shape, _util.weights_of(d), path="large", schedule="dynamic")
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
    _util.assert_out_close(gen.bf16_bits(out), ref_out, f"dynamic {shape.name} T={T} {routing} tiles={tiles}")
    check_internal_permutation(layer, desc, layer._ws, ref_ids, shape.E)


@pytest.mark.parametrize("shape,T", [(gen.QWEN36, 4096), (gen.NEMOTRON, 2048), (gen.LARGE_E, 1024)])
def test_dynamic_schedule_full_shapes(shape, T):
    """Sampled rows against the oracle, the whole output against the static schedule, and
    the trace: every CTA of FC1 and FC2 stamps its phases, and their tiles add up."""
    d = _util.device_layer(shape, T, seed=29)
    w = _util.weights_of(d)
    static = moe.MoELayer(shape, w, path="large", schedule="static")
    dyn = moe.MoELayer(shape, w, path="large", schedule="dynamic")
    ref, ref_w, ref_ids, _ = static.forward(d["x"], return_routing=True)
    trace_s = moe.trace_buffer("cuda")
    static.forward(d["x"], trace=trace_s)
    trace_d = moe.trace_buffer("cuda")
    out, tw, ti, _ = dyn.forward(d["x"], return_routing=True, trace=trace_d)
    torch.cuda.synchronize()
    assert moe.get_error(static._ws) == 0 and moe.get_error(dyn._ws) == 0
    assert torch.equal(ti, ref_ids)
    _util.assert_w_close(tw.cpu().numpy(), ref_w.cpu().numpy())
    _util.assert_out_close(gen.bf16_bits(out), gen.bf16_bits(ref), f"dynamic vs static {shape.name} T={T}")
    # sampled rows against the oracle
    rows = np.random.default_rng(T).choice(T, size=8, replace=False).astype(np.int32)
    h = _util.host_copy(d)
    h["router_logits"] = None
    ref_rows, _, _, ref_rids = oracle.forward(shape, h, rows=rows)
    np.testing.assert_array_equal(ti.cpu().numpy()[rows], ref_rids)
    _util.assert_out_close(gen.bf16_bits(out)[rows], ref_rows, f"dynamic {shape.name} T={T} sampled rows")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ts = trace_s.view(3, moe.TRACE_MAX_CTAS, moe.TRACE_FIELDS).cpu().numpy()
    td = trace_d.view(3, moe.TRACE_MAX_CTAS, moe.TRACE_FIELDS).cpu().numpy()
    for k in (1, 2):  # FC1, FC2
        assert (td[k, :sms, 0] > 0).all() and (td[k, :sms, 4] >= td[k, :sms, 0]).all()
        assert td[k, :sms, 5].sum() == ts[k, :sms, 5].sum(), "the dynamic schedule takes every tile once"

