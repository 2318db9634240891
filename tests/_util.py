"""Helpers for the GPU parity tests: device inputs from the seeded generator, host
copies for the oracle, and the comparison rules (tolerances of the layer contract)."""
import numpy as np
import torch

import oracle
from mixture_experts_layer_35_b200 import inputs as inp_mod

# Layer-output tolerance of the contract: max |gpu - ref| <= 1e-2 max|ref| and
# mean |gpu - ref| <= 1e-3 max|ref|.  Routing weights: 1e-6 relative.
OUT_MAX_REL = 1e-2
OUT_MEAN_REL = 1e-3
W_REL = 1e-6


def device_layer(shape, T, seed=0, routing="router", device="cuda", **kw):
    """Inputs drawn on the device (fast for full-size weights); ``kw``: the generator's
    x_mode / shared_gate / shared_out options."""
    return inp_mod.make_layer(shape, T, seed=seed, device=device, routing=routing, **kw)


def host_copy(d):
    return inp_mod.to_numpy_inputs(d)


def weights_of(d):
    return {k: d[k] for k in ("router_w", "bias", "w13", "w2", "ws13", "ws2", "shared_gate") if d.get(k) is not None}


def bits_f64(t):
    if isinstance(t, torch.Tensor):
        t = inp_mod.bf16_bits(t)
    return oracle.bits_to_f64(t)


def assert_out_close(got_bits, ref_bits, what=""):
    g = bits_f64(got_bits)
    r = bits_f64(ref_bits)
    scale = max(np.abs(r).max(), 1e-30)
    err = np.abs(g - r)
    assert err.max() <= OUT_MAX_REL * scale, f"{what}: max err {err.max():.3e} > {OUT_MAX_REL} * {scale:.3e}"
    assert err.mean() <= OUT_MEAN_REL * scale, f"{what}: mean err {err.mean():.3e} > {OUT_MEAN_REL} * {scale:.3e}"
    return err.max() / scale, err.mean() / scale


def assert_w_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= W_REL, f"{what}: routing weight rel err {rel.max():.3e}"


def check_fused_routing(gpu_ids, gpu_w, gpu_logits, ref_ids, ref_w, ref_logits, shape, bias, given_logits):
    """Routing of the fused path: expert ids bit-exact and weights within 1e-6 relative
    on every row.  When the GPU computes the logits, the ones it returns lie within
    1e-5 max|l| of the oracle's FP64-accumulated FP32 logits (the tensor-core router's
    screening logits; the experts near the top-K boundary are re-evaluated in FP64 and
    match the oracle's rounding)."""
    np.testing.assert_array_equal(np.asarray(gpu_ids), np.asarray(ref_ids))
    assert_w_close(gpu_w, ref_w, "routing weights")
    scale = max(np.abs(ref_logits).max(), 1.0)
    lerr = np.abs(np.asarray(gpu_logits, np.float64) - ref_logits).max()
    assert lerr <= 1e-5 * scale, f"router logits err {lerr:.3e} > {1e-5 * scale:.3e}"
    return np.ones(len(ref_ids), bool)
