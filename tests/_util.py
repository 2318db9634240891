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


def device_layer(shape, T, seed=0, routing="router", device="cuda"):
    """Inputs drawn on the device (fast for full-size weights)."""
    return inp_mod.make_layer(shape, T, seed=seed, device=device, routing=routing)


def host_copy(d):
    return inp_mod.to_numpy_inputs(d)


def weights_of(d):
    return {k: d[k] for k in ("router_w", "bias", "w13", "w2", "ws13", "ws2") if d.get(k) is not None}


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


def oracle_keys(logits, shape, bias):
    """Selection keys from the oracle's FP32 logits (for tie margins only)."""
    l = np.asarray(logits, np.float32)
    if shape.score == "sigmoid":
        s = (1.0 / (1.0 + np.exp(-l.astype(np.float64)))).astype(np.float32)
        return s + (np.zeros_like(s) if bias is None else np.asarray(bias, np.float32))
    return l if bias is None else (l + np.asarray(bias, np.float32))


def routing_rows_unique(ref_logits, shape, bias, logit_tol):
    """Rows whose top-K set (and slot order) cannot change under a logit perturbation of
    `logit_tol`: every gap between consecutive keys down to the (K+1)-th exceeds twice
    the induced key perturbation."""
    keys = oracle_keys(ref_logits, shape, bias).astype(np.float64)
    dk = logit_tol * (0.25 if shape.score == "sigmoid" else 1.0)
    srt = -np.sort(-keys, axis=1)[:, :shape.K + 1]
    gaps = srt[:, :-1] - srt[:, 1:]
    return gaps.min(axis=1) > 2 * dk + 1e-12


def check_fused_routing(gpu_ids, gpu_w, gpu_logits, ref_ids, ref_w, ref_logits, shape, bias, given_logits):
    """IDs: bit-exact wherever the selection is unique.  With given logits that is every
    row.  With logits computed on the GPU (FP32 accumulation in a different order than
    the oracle's FP64 sum), rows whose key gaps lie within the logit rounding may
    legitimately differ: there the GPU's choice must still be a valid top-K of the
    oracle's keys up to that rounding.  Returns the mask of rows whose ids match."""
    gpu_ids = np.asarray(gpu_ids)
    ref_ids = np.asarray(ref_ids)
    if given_logits:
        np.testing.assert_array_equal(gpu_ids, ref_ids)
        assert_w_close(gpu_w, ref_w, "routing weights")
        return np.ones(len(ref_ids), bool)
    scale = max(np.abs(ref_logits).max(), 1.0)
    tol = 1e-5 * scale
    lerr = np.abs(np.asarray(gpu_logits, np.float64) - ref_logits).max()
    assert lerr <= tol, f"router logits err {lerr:.3e} > {tol:.3e}"
    unique = routing_rows_unique(ref_logits, shape, bias, tol)
    np.testing.assert_array_equal(gpu_ids[unique], ref_ids[unique])
    same = np.all(gpu_ids == ref_ids, axis=1)
    keys = oracle_keys(ref_logits, shape, bias).astype(np.float64)
    dk = 2 * tol * (0.25 if shape.score == "sigmoid" else 1.0)
    for r in np.nonzero(~same)[0]:
        sel = set(gpu_ids[r].tolist())
        assert len(sel) == shape.K
        kin = min(keys[r, e] for e in sel)
        kout = max((keys[r, e] for e in range(shape.E) if e not in sel), default=-np.inf)
        assert kin >= kout - dk, f"row {r}: GPU selection is not a top-{shape.K} within rounding"
    assert_w_close(gpu_w[same], ref_w[same], "routing weights")
    assert (~same).sum() <= max(2, len(same) // 100)
    return same
