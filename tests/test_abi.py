"""CPU checks of the C ABI: the library loads, exports every function include/moe.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest
import torch

import mixture_experts_layer_35_b200.moe as moe
from mixture_experts_layer_35_b200 import inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert set(names) == set(moe.EXPORTS)
    for n in names:
        assert hasattr(moe.lib(), n), n


def test_status_strings():
    assert moe.status_string(0) == "MOE_OK"
    assert moe.status_string(3) == "MOE_ERR_WORKSPACE"
    assert moe.status_string(99) == "MOE_ERR_UNKNOWN"


FAKE = 1 << 20  # a 16-byte aligned, never-dereferenced address


def _desc(**kw):
    base = dict(T=4, H=256, I=128, E=16, top_k=4, act="swiglu", score="sigmoid", renorm=True, I_shared=128)
    base.update(kw)
    d = moe.make_desc(**base)
    d.router_w, d.w13, d.w2, d.ws13, d.ws2 = FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5
    return d


def _fwd(d, x=FAKE * 6, out=FAKE * 7, ws=None, ws_bytes=0):
    return moe.lib().moe_fused_forward(ctypes.byref(d), x, out, None, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("field,value,status", [
    ("H", 250, moe.MOE_ERR_INVALID_ARG),
    ("I", 4, moe.MOE_ERR_INVALID_ARG),
    ("top_k", 17, moe.MOE_ERR_INVALID_ARG),
    ("top_k", 0, moe.MOE_ERR_INVALID_ARG),
    ("E", 2048, moe.MOE_ERR_UNSUPPORTED),
    ("act", 7, moe.MOE_ERR_INVALID_ARG),
    ("score", 5, moe.MOE_ERR_INVALID_ARG),
    ("path", 9, moe.MOE_ERR_INVALID_ARG),
    ("schedule", 3, moe.MOE_ERR_INVALID_ARG),
    ("schedule", -1, moe.MOE_ERR_INVALID_ARG),
    ("fc1_tile_rows", 96, moe.MOE_ERR_INVALID_ARG),
    ("fc1_tile_rows", 256, moe.MOE_ERR_INVALID_ARG),  # SwiGLU has no 256-row FC1 tile
    ("fc2_tile_rows", 64, moe.MOE_ERR_INVALID_ARG),
    ("T", -1, moe.MOE_ERR_INVALID_ARG),
    ("T", 1 << 20, moe.MOE_ERR_UNSUPPORTED),
    ("I_shared", 12, moe.MOE_ERR_INVALID_ARG),
])
def test_forward_rejects_bad_descriptions(field, value, status):
    d = _desc()
    setattr(d, field, value)
    assert _fwd(d) == status
    assert moe.workspace_size(d) == 0


def test_forward_rejects_missing_or_misaligned_pointers():
    d = _desc()
    d.w13 = None
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG
    d = _desc()
    d.w2 = FAKE + 4
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG
    d = _desc()
    d.router_w = None  # and no router logits
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG
    d = _desc()
    assert _fwd(d, x=FAKE + 2) == moe.MOE_ERR_INVALID_ARG


def test_forward_checks_workspace_before_launch():
    d = _desc()
    need = moe.workspace_size(d)
    assert need > 256
    assert _fwd(d, ws=None, ws_bytes=need) == moe.MOE_ERR_WORKSPACE
    assert _fwd(d, ws=FAKE * 8, ws_bytes=need - 1) == moe.MOE_ERR_WORKSPACE
    assert _fwd(d, ws=FAKE * 8 + 16, ws_bytes=need) == moe.MOE_ERR_WORKSPACE


def test_zero_tokens_is_a_noop():
    d = _desc(T=0)
    assert _fwd(d, ws=None, ws_bytes=0) == moe.MOE_OK
    assert moe.launches(d) == 0


def test_path_selection_and_launch_counts():
    d = _desc(T=4)
    assert moe.select_path(d) == "small"
    assert moe.launches(d) == 4
    d = _desc(T=4096)
    assert moe.select_path(d) == "large"
    assert moe.launches(d) == 7  # prep, router, top-k, permute, fc1, fc2, finalize
    d = _desc(T=4096, E=512, top_k=10)
    assert moe.launches(d) == 9  # prep, router, top-k in three kernels, permute, fc1, fc2, finalize
    d = _desc(T=4096, E=512, top_k=10, score="softmax", renorm=False)
    assert moe.launches(d) == 7  # full softmax keeps the one-kernel top-k
    d = _desc(T=4, path="large")
    assert moe.select_path(d) == "large"
    assert moe.launches(d) == 6  # few-token router (it zeroes the counters), top-k, permute, fc1, fc2, finalize
    d.router_logits = FAKE * 8
    assert moe.launches(d) == 6  # logits given: prep, no router launch
    d = _desc(T=64, path="small")
    assert moe.select_path(d) == "small"
    assert _fwd(d, ws=FAKE * 8, ws_bytes=moe.workspace_size(d)) == moe.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("shape,T,path", [
    ("qwen36", 1, "small"), ("qwen36", 2, "small"), ("qwen36", 4, "large"), ("qwen36", 16, "large"),
    ("nemotron", 1, "large"), ("large_e", 1, "large"), ("tiny", 4, "small"), ("tiny", 16, "small")])
def test_selector_follows_touched_weight_bytes(shape, T, path):
    """The streaming path is chosen while the call's expert weights are at most 104 MB."""
    s = gen.SHORT[shape]
    d = _desc(T=T, H=s.H, I=s.I, E=s.E, top_k=s.K, act=s.act, score=s.score, I_shared=s.I_shared)
    assert moe.select_path(d) == path


def test_router_topk_and_permute_validation():
    L = moe.lib()
    assert L.moe_router_topk(FAKE, 0, 8, 16, 17, 1, None, 1, FAKE, FAKE, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(FAKE, 3, 8, 16, 4, 1, None, 1, FAKE, FAKE, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(FAKE, 0, 8, 2048, 4, 1, None, 1, FAKE, FAKE, None, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_router_topk(None, 0, 0, 16, 4, 1, None, 1, None, None, None, None) == moe.MOE_OK
    assert L.moe_router_topk(FAKE + 8, 1, 8, 16, 4, 1, None, 1, FAKE, FAKE, None, None) == moe.MOE_ERR_INVALID_ARG
    need = moe.permute_workspace_size(8, 4, 16)
    assert L.moe_permute(FAKE, 8, 4, 16, FAKE, FAKE, None, None, need, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_permute(FAKE, 8, 4, 16, FAKE, FAKE, None, FAKE * 8, need - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_permute(FAKE, 8, 40, 16, FAKE, FAKE, None, FAKE * 8, need, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_permute(FAKE, -1, 4, 16, FAKE, FAKE, None, FAKE * 8, need, None) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("act,T,K,E,tiles", [
    ("swiglu", 20, 2, 8, (32, 32)), ("swiglu", 150, 2, 8, (64, 128)), ("swiglu", 300, 2, 8, (128, 192)),
    ("swiglu", 800, 2, 8, (128, 256)), ("relu2", 150, 2, 8, (64, 128)), ("relu2", 300, 2, 8, (128, 192)),
    ("relu2", 800, 2, 8, (256, 256)), ("swiglu", 4096, 8, 256, (128, 192)), ("swiglu", 8192, 8, 256, (128, 256)),
    ("relu2", 4096, 6, 128, (256, 256))])
def test_token_tile_widths(act, T, K, E, tiles):
    """Token rows per grouped-GEMM tile follow the average rows per expert T*K/E."""
    d = _desc(T=T, top_k=K, E=E, act=act, I_shared=0)
    assert moe.token_tiles(d) == tiles


def test_token_tile_widths_can_be_chosen():
    d = _desc(T=4096, top_k=8, E=256, act="swiglu", I_shared=0)
    d.fc1_tile_rows, d.fc2_tile_rows = 64, 256
    assert moe.token_tiles(d) == (64, 256)
    d.fc1_tile_rows = 0
    assert moe.token_tiles(d) == (128, 256)
    assert moe.workspace_size(d) > 0


def test_workspace_regions_lie_inside_the_workspace():
    d = _desc(T=300, top_k=4, E=16)
    need = moe.workspace_size(d)
    seen = []
    for region, nbytes in ((moe.WS_TOPK_IDS, 300 * 4 * 4), (moe.WS_TOPK_W, 300 * 4 * 4), (moe.WS_OFFSETS, 17 * 4),
                           (moe.WS_PERM, 300 * 4 * 4)):
        off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
        assert moe.lib().moe_workspace_region(ctypes.byref(d), region, ctypes.byref(off), ctypes.byref(nb)) == 0
        assert nb.value == nbytes and off.value % 256 == 0 and off.value + nb.value <= need
        seen.append((off.value, off.value + nb.value))
    seen.sort()
    assert all(a[1] <= b[0] for a, b in zip(seen, seen[1:])), "regions overlap"
    off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_region(ctypes.byref(d), 9, ctypes.byref(off), ctypes.byref(nb)) == \
        moe.MOE_ERR_INVALID_ARG


def test_noalloc_get_error_validates_before_any_cuda_call():
    assert moe.lib().moe_noalloc_get_error(None, None) == moe.MOE_ERR_INVALID_ARG


def test_optional_parts_are_validated_on_the_host():
    ws = FAKE * 16
    d = _desc(T=4)
    d.routed_scale = float("nan")
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG
    d = _desc(T=4)
    d.routed_scale = float("inf")
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG
    d = _desc(T=4, I_shared=0)
    d.ws13 = d.ws2 = None
    d.shared_gate_w = FAKE * 9
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG  # a gate needs an internal shared expert
    d = _desc(T=4)
    d.shared_out = FAKE * 9
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG  # caller shared output and internal shared expert
    d = _desc(T=4)
    d.shared_gate_w = FAKE * 9 + 8
    assert _fwd(d) == moe.MOE_ERR_INVALID_ARG  # misaligned
    # output overlapping the input, or partly overlapping the caller's shared output
    d = _desc(T=4, I_shared=0)
    d.ws13 = d.ws2 = None
    assert _fwd(d, x=FAKE * 6, out=FAKE * 6 + 256) == moe.MOE_ERR_INVALID_ARG
    d.shared_out = FAKE * 9
    assert _fwd(d, x=FAKE * 6, out=FAKE * 9 + 512) == moe.MOE_ERR_INVALID_ARG
    # the in-place form (out is the shared output) passes validation and reaches the workspace check
    assert _fwd(d, x=FAKE * 6, out=FAKE * 9) == moe.MOE_ERR_WORKSPACE
    d.routed_scale = 2.5
    assert _fwd(d, x=FAKE * 6, out=FAKE * 9) == moe.MOE_ERR_WORKSPACE


def test_kernel_plan_lists_the_launches_in_order():
    assert moe.kernel_plan(_desc(T=4)) == ["router", "route", "fc1", "fc2"]
    assert moe.kernel_plan(_desc(T=4096)) == ["prep", "router", "topk", "permute", "fc1", "fc2", "finalize"]
    assert moe.kernel_plan(_desc(T=4096, E=512, top_k=10)) == ["prep", "router", "topk", "refine", "select",
                                                              "permute", "fc1", "fc2", "finalize"]
    assert moe.kernel_plan(_desc(T=64, path="large")) == ["router", "topk", "permute", "fc1", "fc2", "finalize"]
    assert moe.kernel_plan(_desc(T=65, path="large")) == ["prep", "router", "topk", "permute", "fc1", "fc2",
                                                         "finalize"]
    d = _desc(T=16, path="large")
    d.router_logits = FAKE * 8
    assert moe.kernel_plan(d) == ["prep", "topk", "permute", "fc1", "fc2", "finalize"]
    for T in (1, 16, 64, 300, 4096):
        d = _desc(T=T, path="large")
        assert len(moe.kernel_plan(d)) == moe.launches(d)


def test_trace_summary_on_a_synthetic_trace():
    """The host summary of a phase trace (microseconds from %globaltimer nanoseconds):
    launch skew, median input wait and load span, tail, kernel span and units per CTA;
    rows of CTAs that did not run (zero entry stamp) are left out."""
    t = torch.zeros(3 * moe.TRACE_MAX_CTAS * moe.TRACE_FIELDS, dtype=torch.int64)
    v = t.view(3, moe.TRACE_MAX_CTAS, moe.TRACE_FIELDS)
    # FC1 (block 1): three CTAs, entry / ready / loads done / stores done / exit / units
    v[1, 0, :6] = torch.tensor([1000, 3000, 13000, 14000, 20000, 4])
    v[1, 1, :6] = torch.tensor([2000, 3000, 15000, 16000, 22000, 5])
    v[1, 2, :6] = torch.tensor([1000, 4000, 12000, 13000, 18000, 4])
    s = moe.trace_summary(t, 4)
    assert set(s) == {"fc1"}
    f = s["fc1"]
    assert f["ctas"] == 3
    assert f["launch_skew_us"] == 1.0
    assert f["input_wait_us_median"] == 2.0  # waits 2, 1, 3 us
    assert f["load_span_us_median"] == 10.0  # spans 10, 12, 8 us
    assert f["tail_us"] == 4.0 and f["kernel_us"] == 21.0
    assert f["units_min_max"] == [4, 5]
