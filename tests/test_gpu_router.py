"""Router top-k on the GPU against the oracle (the component gate of "Laguna exact M=8
BF16-input router top-k preregistration": changing epochs of bias, raw-byte equality
of expert ids and source indices, repeat determinism, unchanged inputs, K distinct
in-range ids per row, slot*M+row source mapping, designed lower-ID ties)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_35_b200 import inputs
from tests import _util

pytestmark = pytest.mark.gpu
import mixture_experts_layer_35_b200.moe as moe  # noqa: E402  (fails loudly if the library is missing)

E, K = 256, 10


def _run_case(case, score, logits_dtype, renorm=True):
    lg = case["logits"]
    bias = case["bias"]
    lg_d = lg.cuda()
    b_d = None if bias is None else bias.cuda()
    lg_before = lg_d.clone()
    b_before = None if b_d is None else b_d.clone()
    w, ids, src = moe.router_topk(lg_d, K, score, b_d, renorm)
    w2, ids2, src2 = moe.router_topk(lg_d, K, score, b_d, renorm)
    torch.cuda.synchronize()
    # repeat determinism and unchanged inputs
    assert torch.equal(w.view(torch.int32), w2.view(torch.int32))
    assert torch.equal(ids, ids2) and torch.equal(src, src2)
    assert torch.equal(lg_d.view(torch.int16) if lg_d.dtype == torch.bfloat16 else lg_d,
                       lg_before.view(torch.int16) if lg_d.dtype == torch.bfloat16 else lg_before)
    if b_d is not None:
        assert torch.equal(b_d, b_before)
    is_bf16 = logits_dtype == "bf16"
    host_lg = inputs.bf16_bits(lg) if is_bf16 else lg.numpy()
    rw, rids, rsrc = oracle.topk(host_lg, K, score, None if bias is None else bias.numpy(), renorm,
                                 logits_bf16=is_bf16)
    gids, gsrc, gw = ids.cpu().numpy(), src.cpu().numpy(), w.cpu().numpy()
    # raw-byte equality of ids and source indices
    assert gids.tobytes() == rids.tobytes()
    assert gsrc.tobytes() == rsrc.tobytes()
    _util.assert_w_close(gw, rw)
    M = lg.shape[0]
    assert ((gids >= 0) & (gids < E)).all()
    assert all(len(set(r)) == K for r in gids.tolist())
    np.testing.assert_array_equal(gsrc, np.arange(K)[None, :] * M + np.arange(M)[:, None])
    return (gw == rw).mean()


@pytest.mark.parametrize("M,epochs", [(1, 100), (8, 100), (64, 100), (4096, 10)])
def test_router_topk_changing_bias_epochs(M, epochs):
    exact = []
    for ep in range(epochs):
        mode = ("random", "zero", "straddle")[ep % 3]
        case = inputs.make_router_case(M, E, K, seed=1000 * M + ep, bias_mode=mode)
        exact.append(_run_case(case, "sigmoid", "bf16"))
        if mode == "straddle":  # the tied pair shares slot K: the lower id must win it
            i, j = case["pair"]
            w, ids, _ = moe.router_topk(case["logits"].cuda(), K, "sigmoid", case["bias"].cuda())
            ids = ids.cpu().numpy()
            for r in case["tie_rows"].tolist():
                assert i in ids[r] and j not in ids[r]
    assert np.mean(exact) > 0.999


@pytest.mark.parametrize("M", [1, 64, 4096])
def test_router_topk_fp32_logits_and_softmax(M):
    for ep, (score, mode) in enumerate([("sigmoid", "random"), ("softmax", "none"), ("softmax", "zero"),
                                        ("sigmoid", "zero")]):
        case = inputs.make_router_case(M, E, K, seed=77 + ep, bias_mode=mode, logits_dtype="fp32")
        _run_case(case, score, "fp32")
        _run_case(case, score, "fp32", renorm=False)


@pytest.mark.parametrize("E_,K_", [(16, 4), (8, 8), (40, 3), (512, 10), (1024, 32), (1, 1)])
def test_router_topk_other_shapes(E_, K_):
    g = torch.Generator().manual_seed(E_ * 31 + K_)
    lg = torch.randn((37, E_), generator=g)
    bias = torch.randn((E_,), generator=g) * 0.5
    w, ids, src = moe.router_topk(lg.cuda(), K_, "sigmoid", bias.cuda())
    rw, rids, rsrc = oracle.topk(lg.numpy(), K_, "sigmoid", bias.numpy())
    assert ids.cpu().numpy().tobytes() == rids.tobytes()
    _util.assert_w_close(w.cpu().numpy(), rw)


def test_router_topk_golden_ties():
    from tests import _golden
    fx = _golden.load("router_ties.json")
    c0, c1 = fx["cases"]
    w, ids, _ = moe.router_topk(torch.tensor(c0["logits"]).cuda(), 3, "softmax")
    assert ids.cpu().tolist() == c0["K3_ids"]
    w, ids, _ = moe.router_topk(torch.tensor(c0["logits"]).cuda(), 4, "softmax")
    assert ids.cpu().tolist() == c0["K4_ids"]
    w, ids, _ = moe.router_topk(torch.tensor(c1["logits"]).cuda(), 2, "sigmoid", torch.tensor(c1["bias"]).cuda())
    assert ids.cpu().tolist() == c1["K2_ids"]


def test_router_topk_empty():
    lg = torch.empty((0, 16), device="cuda")
    w, ids, src = moe.router_topk(lg, 4, "sigmoid")
    assert w.shape == (0, 4)
