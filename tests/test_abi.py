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


# ---------------------------------------------------------------- expert parallelism (host checks)


def _mixtral_like(**kw):
    base = dict(d_model=4096, n_routed=8, top_k=2, moe_intermediate_size=14336, renormalize=True)
    base.update(kw)
    return moe.make_config(**base)


def test_ep_workspace_size_checks_the_group():
    cfg = _mixtral_like()
    one = moe.moe_ep_workspace_size(cfg, 1, 64, 128)
    eight = moe.moe_ep_workspace_size(cfg, 8, 64, 128)
    assert one > 0 and eight > 0
    # more receive rows need more h for the owned experts
    assert moe.moe_ep_workspace_size(cfg, 2, 64, 4096) > moe.moe_ep_workspace_size(cfg, 2, 64, 128)
    for world, recv, code in [(3, 128, moe.MOE_ERR_INVALID_ARG),     # 8 experts over 3 ranks
                              (16, 128, moe.MOE_ERR_UNSUPPORTED),    # above MOE_EP_MAX_RANKS
                              (0, 128, moe.MOE_ERR_INVALID_ARG),
                              (2, 0, moe.MOE_ERR_INVALID_ARG)]:      # no receive rows
        with pytest.raises(moe.MoeError) as e:
            moe.moe_ep_workspace_size(cfg, world, 64, recv)
        assert e.value.status == code


def test_ep_recv_rows_bound():
    cfg = _mixtral_like()
    # a token holds at most min(k, E / world) of one owner's experts
    assert moe.moe_ep_recv_rows_bound(cfg, 2, [100, 50]) == 150 * 2
    assert moe.moe_ep_recv_rows_bound(cfg, 8, [100, 50]) == 150 * 1
    assert moe.moe_ep_recv_rows_bound(cfg, 4, [0, 0]) == 1


def _group(world, recv_rows=128, flags=True):
    addr = lambda q, base: base + 4096 * q  # 16-byte aligned stand-in addresses, never dereferenced
    return moe.make_ep_group(recv_rows, [addr(q, 1 << 20) for q in range(world)],
                             [addr(q, 2 << 20) for q in range(world)], [addr(q, 3 << 20) for q in range(world)],
                             [addr(q, 4 << 20) for q in range(world)] if flags else None)


def test_ep_layer_forward_rejects_bad_groups_before_any_launch():
    lib = moe.lib_handle()
    cfg = _mixtral_like()
    cap = _mixtral_like(cap_policy="drop", capacity_factor=1.0)
    rank = (moe.moe_ep_rank * 2)()
    call = lambda c, g, first, num: lib.moe_ep_layer_forward(ctypes.byref(c), ctypes.byref(g), first, num, rank, None)
    assert call(cap, _group(2), 0, 2) == moe.MOE_ERR_UNSUPPORTED         # capacity under expert parallelism
    assert call(cfg, _group(2), 0, 3) == moe.MOE_ERR_INVALID_ARG        # more ranks than the group
    assert call(cfg, _group(2), 1, 2) == moe.MOE_ERR_INVALID_ARG        # range past the group
    assert call(cfg, _group(2, flags=False), 0, 1) == moe.MOE_ERR_INVALID_ARG  # one rank needs flag words
    assert call(cfg, _group(2, recv_rows=0), 0, 2) == moe.MOE_ERR_INVALID_ARG
    g = _group(2)
    g.recv_x[1] = (1 << 20) + 4                                          # misaligned receive buffer
    assert call(cfg, g, 0, 2) == moe.MOE_ERR_INVALID_ARG
    g = _group(2)
    g.world = 9
    assert call(cfg, g, 0, 1) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_ep_layer_forward(ctypes.byref(cfg), None, 0, 1, rank, None) == moe.MOE_ERR_INVALID_ARG


def test_ep_group_marshalling():
    g = _group(3, recv_rows=77)
    assert g.world == 3 and g.recv_rows == 77
    assert [g.recv_x[q] for q in range(3)] == [(1 << 20) + 4096 * q for q in range(3)]
    assert g.flags[2] == (4 << 20) + 8192 and g.recv_x[3] is None
    with pytest.raises(ValueError):
        moe.make_ep_group(1, [1] * 9, [1] * 9, [1] * 9)


def test_ep_handles_reject_bad_arguments():
    lib = moe.lib_handle()
    out = ctypes.c_void_p()
    assert lib.moe_ep_export_handle(None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_open_handle(None, ctypes.byref(out)) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_close_handle(None) == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        moe.moe_ep_open_handle(b"short")


def test_plain_c_caller_links_and_calls_the_host_entry_points(tmp_path):
    """A C99 program that includes only include/moe.h links against the library, resolves every
    entry point and gets the same workspace size as the binding (no GPU needed)."""
    import subprocess

    lib_dir = os.path.dirname(moe.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                           os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"), "-L",
                           lib_dir, "-lmoe_b200", "-Wl,-rpath," + lib_dir, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.strip()
    want = moe.moe_workspace_size(_v3(), 16384)
    assert out == "ok %d" % want, out
