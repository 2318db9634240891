"""Loaders for the hand-derived fixtures under tests/golden/ (no arithmetic of the layer)."""
import json
import os

import numpy as np

from mixture_experts_layer_35_b200.inputs import LayerShape

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32_to_bf16_bits_exact(v):
    """Bit pattern of a value that is exactly representable in BF16 (fixture values are)."""
    a = np.asarray(v, np.float32)
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "fixture value is not exact in BF16"
    return (u >> 16).astype(np.uint16)


def layer_fixture(name):
    """Build (shape, numpy input dict, fixture) from a layer fixture file."""
    fx = load(name)
    H, I, E, K = fx["H"], fx["I"], fx["E"], fx["K"]
    Is = fx.get("I_shared", 0)
    rows1 = 2 * I if fx["act"] == "swiglu" else I
    shape = LayerShape("fixture-" + name, H, I, E, K, fx["act"], fx["score"], fx["renorm"], None, Is)
    x = f32_to_bf16_bits_exact(np.array(fx["x"], np.float32))
    w13 = np.zeros((E, rows1, H), np.float32)
    for e, r, c, v in fx["w1_nonzero"]:
        w13[e, r, c] = v
    w2 = np.zeros((E, H, I), np.float32)
    for e, f, i, v in fx["w2_nonzero"]:
        w2[e, f, i] = v
    inp = {"x": x, "router_w": None, "bias": None,
           "router_logits": np.array(fx["router_logits"], np.float32),
           "w13": f32_to_bf16_bits_exact(w13), "w2": f32_to_bf16_bits_exact(w2),
           "ws13": None, "ws2": None}
    if Is:
        rows1s = 2 * Is if fx["act"] == "swiglu" else Is
        ws13 = np.zeros((rows1s, H), np.float32)
        for r, c, v in fx["ws1_nonzero"]:
            ws13[r, c] = v
        ws2 = np.zeros((H, Is), np.float32)
        for f, i, v in fx["ws2_nonzero"]:
            ws2[f, i] = v
        inp["ws13"] = f32_to_bf16_bits_exact(ws13)
        inp["ws2"] = f32_to_bf16_bits_exact(ws2)
    return shape, inp, fx


def hex_bits(lst):
    return np.array([[int(v, 16) for v in row] for row in lst], np.uint16)
