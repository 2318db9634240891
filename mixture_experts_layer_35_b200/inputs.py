"""Seeded synthetic inputs for the fused MoE layer forward.

This module only draws random numbers and lays out input buffers.  It holds none of
the layer's arithmetic (no scores, no top-k, no GEMM, no activation), so the CPU
oracle and the CUDA path can both be fed from it without sharing any computation.

Shapes follow the workloads of the FlashInfer cuTile fused-MoE pull request
(#4646, "Performance: cuTile versus CUTLASS", benchmark-shape table), the Rocket
GB10 note "Exact-N640 retained tail wins only at Qwen c4" (setup table) and the
router contract of "Laguna exact M=8 BF16-input router top-k preregistration"
(section "Question and arithmetic contract").

Conventions
-----------
* BF16 tensors are returned as ``numpy.uint16`` bit patterns (or torch bf16 tensors
  when generated on a device); FP32 tensors as ``numpy.float32``.
* Every value is drawn in FP32 and rounded to BF16 by torch's round-to-nearest-even
  cast.  ``N(0, v)`` means mean 0 and *variance* v, so weights ~ N(0, 1/fan_in).
* Draw order within one generator: x, router weight, bias, w13 (or w1), w2,
  shared w13 (or w1), shared w2.  The seed fixes every byte.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Static shape and routing mode of one MoE layer."""

    name: str
    H: int            # hidden size
    I: int            # routed-expert intermediate size
    E: int            # number of routed experts
    K: int            # top-k
    act: str          # "swiglu" (w13 = [gate; up]) or "relu2" (w1 only)
    score: str        # "sigmoid" or "softmax"
    renorm: bool      # renormalise the selected weights to sum to one
    bias_var: Optional[float]  # variance of the FP32 selection bias, None = no bias
    I_shared: int     # 0 = no shared expert

    @property
    def m(self) -> int:
        """Weight matrices per expert: 3 for a gated activation, 2 otherwise."""
        return 3 if self.act == "swiglu" else 2


# The five workloads.  Names describe the shape; sizes are those of the pages.
TINY = LayerShape("tiny-H256-I128-E16-top4-swiglu-sigmoid-shared", 256, 128, 16, 4,
                  "swiglu", "sigmoid", True, 0.1, 128)
QWEN36 = LayerShape("qwen3.6-shaped-H2048-I512-E256-top8-swiglu-softmax", 2048, 512, 256, 8,
                    "swiglu", "softmax", True, None, 0)
NEMOTRON = LayerShape("nemotron-shaped-H2688-I1856-E128-top6-relu2-softmax", 2688, 1856, 128, 6,
                      "relu2", "softmax", True, None, 0)
LARGE_E = LayerShape("large-E-H2560-I640-E512-top10-swiglu-sigmoid-shared", 2560, 640, 512, 10,
                     "swiglu", "sigmoid", True, 0.5, 640)

SHAPES = {s.name: s for s in (TINY, QWEN36, NEMOTRON, LARGE_E)}
SHORT = {"tiny": TINY, "qwen36": QWEN36, "nemotron": NEMOTRON, "large_e": LARGE_E}

T_SWEEP = [1 << i for i in range(14)]          # 1, 2, 4, ..., 8192
LARGE_E_T = [4, 8, 16, 256, 4096]


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, var: float, g: torch.Generator, device: str) -> torch.Tensor:
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if var != 1.0:
        t.mul_(math.sqrt(var))
    return t.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """BF16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> torch bf16 tensor on the host."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


X_MODES = ("normal", "scale32", "scale256", "outliers")


def _shape_x(x: torch.Tensor, mode: str, seed: int) -> torch.Tensor:
    """Activation scale of the router stress cases.  ``scale32`` / ``scale256``
    multiply x by a power of two (exact in BF16).  ``outliers`` mimics hidden states with
    outlier channels: 16 seeded columns are multiplied by 64 and 1 % of the tokens
    (at least one) by 16, all powers of two."""
    if mode == "normal":
        return x
    if mode in ("scale32", "scale256"):
        return (x.float() * float(mode[5:])).to(torch.bfloat16)
    if mode == "outliers":
        T, H = x.shape
        g = _gen(seed + 104729, "cpu")
        cols = torch.randperm(H, generator=g)[:16].to(x.device)
        rows = torch.randperm(T, generator=g)[:max(1, T // 100)].to(x.device)
        y = x.float()
        y[:, cols] *= 64.0
        y[rows] *= 16.0
        return y.to(torch.bfloat16)
    raise ValueError(mode)


def make_layer(shape: LayerShape, T: int, seed: int = 0, device: str = "cpu",
               routing: str = "router", zipf_s: float = 1.2, x_mode: str = "normal",
               shared_gate: bool = False, shared_out: bool = False) -> dict:
    """Draw one layer's inputs.

    ``routing="router"``: logits come from the router weight (x . Wr^T on the path).
    ``routing="zipf"``: FP32 router logits are drawn directly as
    ``log p_e + Gumbel(0,1)`` with ``p_e ~ rank_e^-s`` over a seeded random ranking of
    the experts, so that per-token expert choice is Zipf-skewed (load imbalance).
    ``x_mode``: activation scale (see ``_shape_x``); the other draws do not change.
    ``shared_gate``: also a gate row [H] ~ N(0, 1/H) for the shared expert (``shared_gate``);
    ``shared_out``: also a caller-side shared output [T, H] ~ N(0, 1/4) (``shared_out``).
    Both come from their own generators, so the other draws do not change.
    Returns torch tensors on ``device`` (bf16 / fp32).
    """
    H, I, E = shape.H, shape.I, shape.E
    g = _gen(seed, device)
    d = {}
    d["x"] = _shape_x(_normal_bf16((T, H), 1.0, g, device), x_mode, seed)
    d["router_w"] = _normal_bf16((E, H), 1.0 / H, g, device)
    if shape.bias_var is not None:
        d["bias"] = torch.randn((E,), generator=g, device=device) * math.sqrt(shape.bias_var)
    else:
        d["bias"] = None
    rows1 = 2 * I if shape.act == "swiglu" else I
    d["w13"] = _normal_bf16((E, rows1, H), 1.0 / H, g, device)
    d["w2"] = _normal_bf16((E, H, I), 1.0 / I, g, device)
    if shape.I_shared:
        Is = shape.I_shared
        rows1s = 2 * Is if shape.act == "swiglu" else Is
        d["ws13"] = _normal_bf16((rows1s, H), 1.0 / H, g, device)
        d["ws2"] = _normal_bf16((H, Is), 1.0 / Is, g, device)
    else:
        d["ws13"] = None
        d["ws2"] = None
    d["router_logits"] = None
    if routing == "zipf":
        gz = _gen(seed + 7919, device)
        ranks = torch.randperm(E, generator=gz, device=device).to(torch.float64) + 1.0
        logp = -zipf_s * torch.log(ranks)
        logp = logp - torch.logsumexp(logp, 0)
        u = torch.rand((T, E), generator=gz, device=device, dtype=torch.float64)
        u = u.clamp_(min=1e-300)
        gumbel = -torch.log(-torch.log(u))
        d["router_logits"] = (logp[None, :] + gumbel).to(torch.float32)
    elif routing != "router":
        raise ValueError(routing)
    d["shared_gate"] = _normal_bf16((H,), 1.0 / H, _gen(seed + 7717, device), device) if shared_gate else None
    d["shared_out"] = _normal_bf16((T, H), 0.25, _gen(seed + 6007, device), device) if shared_out else None
    return d


def make_router_case(M: int, E: int = 256, K: int = 10, seed: int = 0,
                     bias_mode: str = "random", tie_frac: float = 0.1,
                     logits_dtype: str = "bf16") -> dict:
    """One epoch of the router top-k gate: BF16 (or FP32) logits ~ N(0,1) and a bias.

    ``bias_mode``:
      * ``"random"``: FP32 bias ~ N(0, 0.5); one expert pair (i < j) gets b_j := b_i and
        in ~``tie_frac`` of the rows l_j := l_i, an exact key tie somewhere in the row.
      * ``"zero"``: all-zero bias; in tie rows, half of them copy the logit ranked K-th
        (by raw value) onto the one ranked (K+1)-th (a tie across the slot boundary),
        the other half copy one of the top-K logits onto another top-K expert.
      * ``"straddle"``: K-1 experts get bias +10, a pair (i < j) gets bias +6, the rest
        N(0, 0.5) clipped to [-3, 3]; tie rows set l_j := l_i, so the pair ties for the
        last slot and the lower ID must win it.
      * ``"none"``: no bias tensor (softmax-style routing on raw logits).
    Host tensors; logits bf16 or fp32, bias fp32 or None, plus the tie rows and pair.
    """
    g = _gen(seed, "cpu")
    logits = torch.randn((M, E), generator=g, dtype=torch.float32)
    if logits_dtype == "bf16":
        logits = logits.to(torch.bfloat16)
    n_tie = max(1, int(round(tie_frac * M))) if tie_frac > 0 else 0
    tie_rows = torch.randperm(M, generator=g)[:n_tie].sort().values
    pair = torch.randperm(E, generator=g)[:2].sort().values
    i, j = int(pair[0]), int(pair[1])
    bias = None
    if bias_mode == "random":
        bias = torch.randn((E,), generator=g) * math.sqrt(0.5)
        bias[j] = bias[i]
        for r in tie_rows.tolist():
            logits[r, j] = logits[r, i]
    elif bias_mode == "zero":
        bias = torch.zeros((E,), dtype=torch.float32)
        for n, r in enumerate(tie_rows.tolist()):
            order = torch.argsort(logits[r].float(), descending=True, stable=True)
            if n % 2 == 0:
                logits[r, order[K]] = logits[r, order[K - 1]]
            else:
                a, b = int(order[0]), int(order[min(K - 1, 3)])
                logits[r, max(a, b)] = logits[r, min(a, b)]
    elif bias_mode == "straddle":
        bias = (torch.randn((E,), generator=g) * math.sqrt(0.5)).clamp_(-3.0, 3.0)
        rest = [e for e in torch.randperm(E, generator=g).tolist() if e not in (i, j)]
        for e in rest[:K - 1]:
            bias[e] = 10.0
        bias[i] = 6.0
        bias[j] = 6.0
        for r in tie_rows.tolist():
            logits[r, j] = logits[r, i]
    elif bias_mode == "none":
        bias = None
    else:
        raise ValueError(bias_mode)
    return {"logits": logits, "bias": bias, "tie_rows": tie_rows, "pair": (i, j)}


def to_numpy_inputs(d: dict) -> dict:
    """Host numpy view of a ``make_layer`` dict: bf16 -> uint16 bits, fp32 -> float32."""
    out = {}
    for k, v in d.items():
        if v is None:
            out[k] = None
        elif v.dtype == torch.bfloat16:
            out[k] = bf16_bits(v)
        else:
            out[k] = v.detach().to("cpu").contiguous().numpy()
    return out
