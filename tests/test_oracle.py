"""Pins of the CPU oracle against things other than itself: hand-derived fixtures,
closed forms, brute force over all subsets, high-precision references and library
routines (torch float64 matmul, numpy lexsort).  CPU only."""
import itertools
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_35_b200.inputs import LayerShape, bf16_bits
from tests import _golden

getcontext().prec = 80


# ---------------------------------------------------------------- number formats

def test_bf16_rounding_golden():
    fx = _golden.load("bf16_rounding.json")
    for c in fx["cases"]:
        assert oracle.double_to_bf16(float(c["value"])) == int(c["bits"], 16), c


def test_bf16_rounding_matches_torch_from_float32():
    """From an FP32 value, RNE to BF16 is a single rounding: torch's cast must agree."""
    g = torch.Generator().manual_seed(1)
    v = torch.cat([torch.randn(20000, generator=g) * 10.0 ** torch.randint(-30, 30, (20000,), generator=g).float(),
                   torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 65504.0, 1e-38, -1e-39])])
    v = v[torch.isfinite(v)]
    ref = bf16_bits(v.to(torch.bfloat16))
    got = np.array([oracle.double_to_bf16(float(a)) for a in v.tolist()], np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_bf16_rounding_half_step_property():
    """|v - round(v)| <= half a BF16 step, exact halves go to the even neighbour."""
    rng = np.random.default_rng(2)
    for v in rng.standard_normal(3000) * 100.0:
        b = oracle.double_to_bf16(float(v))
        r = oracle.bf16_to_double(b)
        e = math.frexp(abs(v))[1]
        step = 2.0 ** (e - 8)
        assert abs(r - v) <= step / 2
        if abs(abs(r - v) - step / 2) == 0:
            assert b % 2 == 0


def _sigmoid_f32_exact(l):
    """Correctly rounded FP32 sigmoid from an 80-digit decimal evaluation."""
    d = Decimal(1) / (Decimal(1) + (-Decimal(float(l))).exp())
    f = np.float32(float(d))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    return min(cands, key=lambda c: (abs(Decimal(float(c)) - d), int(np.float32(c).view(np.uint32)) & 1))


def test_sigmoid_is_correctly_rounded():
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(3000) * 3, rng.uniform(-30, 30, 500),
                           [0.0, -0.0, 1e-30, -1e-30, 16.0, -16.0, 88.0, -88.0]]).astype(np.float32)
    for l in vals:
        assert np.float32(oracle.sigmoid_f32(float(l))) == _sigmoid_f32_exact(l), l
    assert oracle.sigmoid_f32(0.0) == 0.5


def test_router_logits_match_float64_matmul():
    g = torch.Generator().manual_seed(4)
    x = torch.randn(5, 96, generator=g).to(torch.bfloat16)
    w = (torch.randn(12, 96, generator=g) / 10).to(torch.bfloat16)
    got = oracle.router_logits(bf16_bits(x), bf16_bits(w))
    ref = (x.double() @ w.double().T).float().numpy()
    ulp = np.abs(np.spacing(ref))
    assert np.all(np.abs(got - ref) <= ulp)
    assert np.mean(got == ref) > 0.99


# ---------------------------------------------------------------- router top-k

def _keys(logits, score, bias):
    if score == "softmax":
        return logits.astype(np.float32) if bias is None else (logits + bias).astype(np.float32)
    s = np.array([_sigmoid_f32_exact(v) for v in logits], np.float32)
    b = np.zeros_like(s) if bias is None else bias.astype(np.float32)
    return (s + b).astype(np.float32)


def _brute_force_topk(key, K):
    E = len(key)
    better = lambda i, j: key[i] > key[j] or (key[i] == key[j] and i < j)
    winners = [S for S in itertools.combinations(range(E), K)
               if all(better(i, j) for i in S for j in range(E) if j not in S)]
    assert len(winners) == 1
    return sorted(winners[0], key=lambda i: (-float(key[i]), i))


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
@pytest.mark.parametrize("E,K", [(5, 1), (6, 2), (8, 3), (10, 4), (12, 4)])
def test_topk_brute_force_with_ties(score, E, K):
    rng = np.random.default_rng(E * 10 + K)
    grid = np.array([-1.0, -0.5, 0.0, 0.5, 1.0, 2.0], np.float32)
    for trial in range(20):
        lg = rng.choice(grid, size=(3, E)).astype(np.float32)
        bias = None
        if trial % 2 == 1:
            bias = rng.choice(np.array([0.0, 0.25, -0.25], np.float32), size=E).astype(np.float32)
        w, ids, src = oracle.topk(lg, K, score, bias)
        for m in range(lg.shape[0]):
            assert list(ids[m]) == _brute_force_topk(_keys(lg[m], score, bias), K)


def test_topk_golden_ties():
    fx = _golden.load("router_ties.json")
    c0, c1 = fx["cases"]
    lg = np.array(c0["logits"], np.float32)
    w, ids, _ = oracle.topk(lg, 3, "softmax")
    assert ids.tolist() == c0["K3_ids"]
    np.testing.assert_array_equal(w, np.float32(1.0 / 3.0))
    w, ids, _ = oracle.topk(lg, 4, "softmax")
    assert ids.tolist() == c0["K4_ids"]
    d = 3.0 + math.exp(-1.0)
    np.testing.assert_allclose(w[0], [1 / d, 1 / d, 1 / d, math.exp(-1.0) / d], rtol=1e-7)
    lg = np.array(c1["logits"], np.float32)
    w, ids, _ = oracle.topk(lg, 2, "sigmoid", np.array(c1["bias"], np.float32))
    assert ids.tolist() == c1["K2_ids"]
    s05, s1 = 1 / (1 + math.exp(-0.5)), 1 / (1 + math.exp(-1.0))
    np.testing.assert_allclose(w[0], [s05 / (s05 + s1), s1 / (s05 + s1)], rtol=1e-6)


def test_topk_source_index_mapping():
    M, K = _golden.load("router_ties.json")["src_mapping"]["M"], 10
    lg = np.random.default_rng(5).standard_normal((M, 32)).astype(np.float32)
    _, _, src = oracle.topk(lg, K, "sigmoid")
    for m in range(M):
        for k in range(K):
            assert src[m, k] == k * 8 + m


def test_topk_weights_closed_forms():
    rng = np.random.default_rng(6)
    lg = rng.standard_normal((50, 16)).astype(np.float32)
    bias = (rng.standard_normal(16) * 0.7).astype(np.float32)
    for score in ("sigmoid", "softmax"):
        w, ids, _ = oracle.topk(lg, 5, score, bias if score == "sigmoid" else None, renorm=True)
        np.testing.assert_allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)
        w1, _, _ = oracle.topk(lg, 1, score, None, renorm=True)
        np.testing.assert_array_equal(w1, 1.0)
    # sigmoid without renorm: the unbiased FP32 score itself
    w, ids, _ = oracle.topk(lg, 4, "sigmoid", bias, renorm=False)
    for m in range(lg.shape[0]):
        for k in range(4):
            assert w[m, k] == _sigmoid_f32_exact(lg[m, ids[m, k]])
    # softmax with K = E: the full softmax, in descending-logit slot order
    w, ids, _ = oracle.topk(lg, 16, "softmax", None, renorm=True)
    ref = torch.softmax(torch.from_numpy(lg).double(), dim=1).numpy()
    np.testing.assert_allclose(w, np.take_along_axis(ref, ids, 1), rtol=1e-6)
    w2, _, _ = oracle.topk(lg, 16, "softmax", None, renorm=False)
    np.testing.assert_allclose(w2, w, rtol=1e-6)


def test_topk_bias_only_selects():
    """The bias moves the selection but never the weights of the experts it selects."""
    lg = np.array([[0.0, 1.0, 2.0, 3.0]], np.float32)
    bias = np.array([10.0, 0.0, 0.0, -10.0], np.float32)
    w, ids, _ = oracle.topk(lg, 2, "sigmoid", bias, renorm=False)
    assert ids.tolist() == [[0, 2]]
    assert w[0, 0] == _sigmoid_f32_exact(np.float32(0.0)) and w[0, 1] == _sigmoid_f32_exact(np.float32(2.0))


# ---------------------------------------------------------------- permutation

def test_permute_matches_lexsort():
    rng = np.random.default_rng(7)
    for M, K, E in [(1, 1, 1), (5, 3, 8), (64, 8, 256), (300, 6, 128), (17, 10, 512)]:
        ids = np.stack([rng.permutation(E)[:K] for _ in range(M)]).astype(np.int32)
        offsets, perm, inv = oracle.permute(ids, E)
        t = np.repeat(np.arange(M), K)
        k = np.tile(np.arange(K), M)
        e = ids.reshape(-1)
        order = np.lexsort((t, e))
        np.testing.assert_array_equal(perm, (k * M + t)[order])
        np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(e, minlength=E))]))
        np.testing.assert_array_equal(inv[perm], np.arange(M * K))


def test_permute_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 9]], np.int32), 8)
    with pytest.raises(ValueError):
        oracle.permute(np.array([[-1, 2]], np.int32), 8)


# ---------------------------------------------------------------- layer forward

def _rand_bits(shape, scale, g):
    return bf16_bits((torch.randn(shape, generator=g) * scale).to(torch.bfloat16))


def _dense_mlp_ref(x, w13, w2, act, I):
    """torch float64 composition of one expert on all tokens; h rounded to BF16."""
    g = x @ w13.T
    if act == "swiglu":
        a = torch.nn.functional.silu(g[:, :I]) * g[:, I:]
    else:
        a = torch.relu(g) ** 2
    h = a.float().to(torch.bfloat16).double()
    return h @ w2.T


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_forward_single_expert_is_dense_mlp(act):
    H, I, T = 48, 24, 6
    shape = LayerShape("dense", H, I, 1, 1, act, "softmax", True, None, 0)
    g = torch.Generator().manual_seed(8)
    rows1 = 2 * I if act == "swiglu" else I
    inp = {"x": _rand_bits((T, H), 1.0, g), "router_w": _rand_bits((1, H), 0.2, g), "bias": None,
           "router_logits": None, "w13": _rand_bits((1, rows1, H), H ** -0.5, g),
           "w2": _rand_bits((1, H, I), I ** -0.5, g), "ws13": None, "ws2": None}
    out, lg, w, ids = oracle.forward(shape, inp)
    assert (ids == 0).all() and (w == 1.0).all()
    ref = _dense_mlp_ref(torch.from_numpy(oracle.bits_to_f64(inp["x"])),
                         torch.from_numpy(oracle.bits_to_f64(inp["w13"][0])),
                         torch.from_numpy(oracle.bits_to_f64(inp["w2"][0])), act, I).numpy()
    got = oracle.bits_to_f64(out)
    err = np.abs(got - ref)
    assert err.max() <= 4e-3 * np.abs(ref).max()


def test_forward_full_softmax_mixture_with_shared():
    """K = E with softmax renorm is the full softmax mixture; the shared expert is added
    after rounding the routed sum (checked against a torch float64 composition)."""
    H, I, E, T = 32, 16, 4, 5
    shape = LayerShape("mix", H, I, E, E, "swiglu", "softmax", True, None, I)
    g = torch.Generator().manual_seed(9)
    inp = {"x": _rand_bits((T, H), 1.0, g), "router_w": _rand_bits((E, H), 0.3, g), "bias": None,
           "router_logits": None, "w13": _rand_bits((E, 2 * I, H), H ** -0.5, g),
           "w2": _rand_bits((E, H, I), I ** -0.5, g), "ws13": _rand_bits((2 * I, H), H ** -0.5, g),
           "ws2": _rand_bits((H, I), I ** -0.5, g)}
    out, lg, w, ids = oracle.forward(shape, inp)
    x = torch.from_numpy(oracle.bits_to_f64(inp["x"]))
    logits = (x @ torch.from_numpy(oracle.bits_to_f64(inp["router_w"])).T).float().double()
    p = torch.softmax(logits, 1)
    routed = sum(p[:, e:e + 1] * _dense_mlp_ref(x, torch.from_numpy(oracle.bits_to_f64(inp["w13"][e])),
                                                torch.from_numpy(oracle.bits_to_f64(inp["w2"][e])), "swiglu", I)
                 for e in range(E))
    routed = routed.float().to(torch.bfloat16).double()
    shared = _dense_mlp_ref(x, torch.from_numpy(oracle.bits_to_f64(inp["ws13"])),
                            torch.from_numpy(oracle.bits_to_f64(inp["ws2"])), "swiglu", I)
    ref = (routed + shared.float().to(torch.bfloat16).double()).numpy()
    got = oracle.bits_to_f64(out)
    assert np.abs(got - ref).max() <= 1e-2 * np.abs(ref).max()
    assert np.abs(got - ref).mean() <= 1e-3 * np.abs(ref).max()


@pytest.mark.parametrize("name", ["relu2_integer.json", "combine_order.json", "h_rounding.json"])
def test_forward_golden_exact(name):
    shape, inp, fx = _golden.layer_fixture(name)
    out, lg, w, ids = oracle.forward(shape, inp)
    np.testing.assert_array_equal(out, _golden.hex_bits(fx["expected_out_bits"]))
    if "expected_ids" in fx:
        assert ids.tolist() == fx["expected_ids"]
        np.testing.assert_array_equal(w, np.array(fx["expected_w"], np.float32))


def test_forward_linear_in_w2():
    """Doubling every W2 doubles the routed output exactly (powers of two commute with
    BF16 rounding away from overflow/underflow)."""
    H, I, E, K, T = 32, 16, 6, 2, 4
    shape = LayerShape("lin", H, I, E, K, "relu2", "sigmoid", True, None, 0)
    g = torch.Generator().manual_seed(10)
    inp = {"x": _rand_bits((T, H), 1.0, g), "router_w": _rand_bits((E, H), 0.3, g),
           "bias": np.zeros(E, np.float32), "router_logits": None,
           "w13": _rand_bits((E, I, H), H ** -0.5, g), "w2": _rand_bits((E, H, I), I ** -0.5, g),
           "ws13": None, "ws2": None}
    out1, *_ = oracle.forward(shape, inp)
    w2x2 = bf16_bits(torch.from_numpy(oracle.bits_to_f64(inp["w2"]) * 2).to(torch.bfloat16))
    out2, *_ = oracle.forward(shape, dict(inp, w2=w2x2))
    np.testing.assert_array_equal(oracle.bits_to_f64(out2), 2 * oracle.bits_to_f64(out1))


def test_forward_rows_subset_and_given_logits():
    H, I, E, K, T = 32, 16, 8, 3, 7
    shape = LayerShape("sub", H, I, E, K, "swiglu", "sigmoid", True, 0.5, 0)
    g = torch.Generator().manual_seed(11)
    inp = {"x": _rand_bits((T, H), 1.0, g), "router_w": _rand_bits((E, H), 0.3, g),
           "bias": (torch.randn(E, generator=g) * 0.5).numpy(), "router_logits": None,
           "w13": _rand_bits((E, 2 * I, H), H ** -0.5, g), "w2": _rand_bits((E, H, I), I ** -0.5, g),
           "ws13": None, "ws2": None}
    out, lg, w, ids = oracle.forward(shape, inp)
    rows = np.array([6, 0, 3], np.int32)
    o2, l2, w2, i2 = oracle.forward(shape, inp, rows)
    np.testing.assert_array_equal(o2, out[rows])
    np.testing.assert_array_equal(i2, ids[rows])
    o3, l3, w3, i3 = oracle.forward(shape, dict(inp, router_logits=lg, router_w=None))
    np.testing.assert_array_equal(o3, out)
    np.testing.assert_array_equal(lg, oracle.router_logits(inp["x"], inp["router_w"]))
    w4, i4, _ = oracle.topk(lg, K, "sigmoid", inp["bias"])
    np.testing.assert_array_equal(i4, ids)
    np.testing.assert_array_equal(w4, w)


def test_sharded_oracle_equals_one_process():
    from mixture_experts_layer_35_b200 import inputs as gen
    """oracle.parallel runs the same C oracle on token ranges in spawned processes; the
    concatenation must equal the single-process result bit for bit."""
    from oracle import parallel as opar
    shape = gen.TINY
    h = gen.to_numpy_inputs(gen.make_layer(shape, 37, seed=4))
    one = oracle.forward(shape, h)
    rows = np.arange(37, dtype=np.int32)[::-1].copy()
    many = opar.forward_parallel(shape, h, rows, procs=3)
    ref = oracle.forward(shape, h, rows)
    for a, b in zip(many, ref):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(many[0][::-1], one[0])


# ---------------------------------------------------------------- routed scale, shared gate, shared output

def _small_layer_inputs(seed, H=32, I=16, E=6, K=2, shared=True):
    g = torch.Generator().manual_seed(seed)
    inp = {"x": _rand_bits((5, H), 1.0, g), "router_w": _rand_bits((E, H), 0.3, g),
           "bias": (torch.randn(E, generator=g) * 0.3).numpy(), "router_logits": None,
           "w13": _rand_bits((E, 2 * I, H), H ** -0.5, g), "w2": _rand_bits((E, H, I), I ** -0.5, g),
           "ws13": _rand_bits((2 * I, H), H ** -0.5, g) if shared else None,
           "ws2": _rand_bits((H, I), I ** -0.5, g) if shared else None}
    return LayerShape("extras", H, I, E, K, "swiglu", "sigmoid", True, 0.09, I if shared else 0), inp


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_routed_scale_on_a_dense_mlp(act):
    """One expert, K = 1: the routed output is bf16(scale * dense MLP(x)), the dense MLP
    taken from a torch float64 composition ("Laguna ...", "Question and arithmetic
    contract": the configured routed scale multiplies the routed output)."""
    H, I, T, scale = 40, 24, 6, 2.5
    shape = LayerShape("dense", H, I, 1, 1, act, "softmax", True, None, 0)
    g = torch.Generator().manual_seed(12)
    rows1 = 2 * I if act == "swiglu" else I
    inp = {"x": _rand_bits((T, H), 1.0, g), "router_w": _rand_bits((1, H), 0.2, g), "bias": None,
           "router_logits": None, "w13": _rand_bits((1, rows1, H), H ** -0.5, g),
           "w2": _rand_bits((1, H, I), I ** -0.5, g), "ws13": None, "ws2": None}
    out, *_ = oracle.forward(shape, inp, routed_scale=scale)
    ref = scale * _dense_mlp_ref(torch.from_numpy(oracle.bits_to_f64(inp["x"])),
                                 torch.from_numpy(oracle.bits_to_f64(inp["w13"][0])),
                                 torch.from_numpy(oracle.bits_to_f64(inp["w2"][0])), act, I).numpy()
    got = oracle.bits_to_f64(out)
    assert np.abs(got - ref).max() <= 4e-3 * np.abs(ref).max()
    assert not np.array_equal(out, oracle.forward(shape, inp)[0])


def test_routed_scale_two_is_w2_doubled():
    """A routed scale of 2 equals doubling every routed W2 (exact in BF16), bit for bit,
    with the shared expert unchanged."""
    shape, inp = _small_layer_inputs(13)
    w2x2 = bf16_bits(torch.from_numpy(oracle.bits_to_f64(inp["w2"]) * 2).to(torch.bfloat16))
    a, *_ = oracle.forward(shape, inp, routed_scale=2.0)
    b, *_ = oracle.forward(shape, dict(inp, w2=w2x2))
    np.testing.assert_array_equal(a, b)


def test_shared_gate_special_values():
    """A zero gate row gives sigmoid(0) = 1/2, the same bits as halving the shared W2
    (exact); a gate logit far above 0 gives sigmoid = 1.0 in FP32, the ungated bits."""
    shape, inp = _small_layer_inputs(14)
    H = shape.H
    zero = np.zeros(H, np.uint16)
    half = bf16_bits(torch.from_numpy(oracle.bits_to_f64(inp["ws2"]) / 2).to(torch.bfloat16))
    a, *_ = oracle.forward(shape, dict(inp, shared_gate=zero))
    b, *_ = oracle.forward(shape, dict(inp, ws2=half))
    np.testing.assert_array_equal(a, b)
    # gate row = 2^7 * sign(x) on every column of every token: logit >= 128 * min |x| sum
    x = oracle.bits_to_f64(inp["x"])
    assert (np.abs(x).sum(1) * 128 > 120).all()
    big = np.full(H, 0x4300, np.uint16)  # 128.0
    xs = np.abs(x)
    sign_x = bf16_bits(torch.from_numpy(np.abs(x) / np.where(xs > 0, xs, 1.0)).to(torch.bfloat16))
    inp_pos = dict(inp, x=sign_x)  # every x entry +1 or 0: gate logit = 128 * (count of nonzero) >= 128
    c, *_ = oracle.forward(shape, dict(inp_pos, shared_gate=big))
    d, *_ = oracle.forward(shape, inp_pos)
    np.testing.assert_array_equal(c, d)


def test_shared_gate_against_torch_composition():
    """The gated shared output is bf16(sigmoid(fp32(x . w_g)) * shared FFN(x)) added after
    the routed rounding (torch float64 composition, the same tolerance as the layer)."""
    shape, inp = _small_layer_inputs(15, E=4, K=4)
    g = torch.Generator().manual_seed(16)
    gate = _rand_bits((shape.H,), 0.4, g)
    with_gate, *_ = oracle.forward(shape, dict(inp, shared_gate=gate))
    no_shared = dict(inp, ws13=None, ws2=None)
    routed, *_ = oracle.forward(LayerShape("r", shape.H, shape.I, shape.E, shape.K, "swiglu", "sigmoid", True, 0.09, 0),
                                no_shared)
    x = torch.from_numpy(oracle.bits_to_f64(inp["x"]))
    lg = (x @ torch.from_numpy(oracle.bits_to_f64(gate))).float().double()
    s = torch.sigmoid(lg).float().double()
    y = _dense_mlp_ref(x, torch.from_numpy(oracle.bits_to_f64(inp["ws13"])),
                       torch.from_numpy(oracle.bits_to_f64(inp["ws2"])), "swiglu", shape.I)
    ys = (s[:, None] * y).float().to(torch.bfloat16).double()
    ref = (torch.from_numpy(oracle.bits_to_f64(routed)) + ys).numpy()
    got = oracle.bits_to_f64(with_gate)
    assert np.abs(got - ref).max() <= 1e-2 * np.abs(ref).max()
    assert np.abs(got - ref).mean() <= 1e-3 * np.abs(ref).max()


@pytest.mark.parametrize("gated", [False, True])
def test_caller_shared_output_equals_internal_shared_expert(gated):
    """The shared output the layer would compute, handed in by the caller instead (the
    "MTP1 isolated gather/shared-add closure" form), gives the same bits: the internal
    shared output is read off a run whose routed W2 is zero (routed sum 0)."""
    shape, inp = _small_layer_inputs(17)
    if gated:
        inp["shared_gate"] = _rand_bits((shape.H,), 0.4, torch.Generator().manual_seed(18))
    zero_w2 = np.zeros_like(inp["w2"])
    ys, *_ = oracle.forward(shape, dict(inp, w2=zero_w2))
    full, *_ = oracle.forward(shape, inp, routed_scale=1.5)
    ext_shape = LayerShape("ext", shape.H, shape.I, shape.E, shape.K, "swiglu", "sigmoid", True, 0.09, 0)
    ext, *_ = oracle.forward(ext_shape, dict(inp, ws13=None, ws2=None, shared_gate=None, shared_out=ys),
                             routed_scale=1.5)
    np.testing.assert_array_equal(ext, full)
