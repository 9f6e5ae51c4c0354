"""The C-ABI library: it loads, exports every symbol include/moe.h declares, and
rejects bad arguments on the host before anything reaches a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

import top_routing_expert_router_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    declared = _declared()
    assert declared, "no declarations found"
    lib = ctypes.CDLL(moe.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(moe.EXPORTS)


def _v3(**kw):
    base = dict(d_model=7168, n_routed=256, top_k=8, moe_intermediate_size=2048, n_shared=1, n_group=8,
                topk_group=4, score_fn="sigmoid", renormalize=True, routed_scaling_factor=2.5)
    base.update(kw)
    return moe.make_config(**base)


def test_workspace_size_valid_and_monotone():
    a = moe.moe_workspace_size(_v3(), 64)
    b = moe.moe_workspace_size(_v3(), 16384)
    assert 0 < a < b
    assert moe.moe_workspace_size(_v3(), 0) > 0


@pytest.mark.parametrize("bad,code", [
    (dict(top_k=300), moe.MOE_ERR_INVALID_ARG),           # k > E
    (dict(n_group=7), moe.MOE_ERR_INVALID_ARG),           # E not divisible by groups
    (dict(topk_group=9), moe.MOE_ERR_INVALID_ARG),        # more kept groups than groups
    (dict(topk_group=1, top_k=40), moe.MOE_ERR_INVALID_ARG),  # kept groups cannot hold k experts
    (dict(d_model=7170), moe.MOE_ERR_UNSUPPORTED),        # rows not 16-byte multiples
    (dict(score_fn="softmax"), moe.MOE_ERR_UNSUPPORTED),  # group limit with softmax
    (dict(n_routed=512, n_group=8), moe.MOE_ERR_UNSUPPORTED),
    (dict(cap_policy="overflow_next"), moe.MOE_ERR_INVALID_ARG),  # no capacity given
])
def test_bad_config_rejected(bad, code):
    with pytest.raises(moe.MoeError) as e:
        moe.moe_workspace_size(_v3(**bad), 16)
    assert e.value.status == code


def test_bad_pointers_rejected_before_any_launch():
    cfg = _v3()
    lib = moe.lib_handle()
    need = moe.moe_workspace_size(cfg, 16)
    w = moe.moe_weights(*([256] * 8))
    # misaligned workspace
    st = lib.moe_layer_forward(ctypes.byref(cfg), 16, 256, ctypes.byref(w), 256, None, None, None, None, 257,
                               need, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    st = lib.moe_layer_forward(ctypes.byref(cfg), 16, 256, ctypes.byref(w), 256, None, None, None, None, 256,
                               need - 1, None)
    assert st == moe.MOE_ERR_WORKSPACE
    # null x
    st = lib.moe_route(ctypes.byref(cfg), 16, None, ctypes.byref(w), 256, 256, None, None, 256, need, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # misaligned output
    st = lib.moe_route(ctypes.byref(cfg), 16, 256, ctypes.byref(w), 260, 256, None, None, 256, need, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # negative n
    st = lib.moe_permute(ctypes.byref(cfg), -1, 256, 256, 256, 256, 256, 256, 256, need, None)
    assert st == moe.MOE_ERR_INVALID_ARG


def test_status_strings():
    for code in range(7):
        assert moe.moe_status_string(code)
    assert moe.moe_status_string(99) == "unknown status"
