"""moe_route_static_scratch: the router for callers that cannot allocate.

Some callers of this library never allocate device memory themselves: a
plug-in that runs inside a serving engine only receives the input and output
buffers the engine's memory planner hands it, and code on a latency-critical
path must not call cudaMalloc because it synchronises the device. Those
callers cannot supply a workspace, so this entry point keeps the router's
scratch in a fixed-size device array that is part of the library.

The array is shared by every call and keeps the previous call's contents, so
each test below routes twice in a row and compares both results with
moe_route run on a caller-provided workspace: same expert indices and counts,
gates within the tolerance of the routing parity tests. This file is named so
that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import top_routing_expert_router_b200 as moe
from synth import workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _outputs(w):
    return (torch.full((w.n, w.top_k), -9, dtype=torch.int32, device="cuda"),
            torch.full((w.n, w.top_k), -9.0, dtype=torch.float32, device="cuda"),
            torch.full((w.n_routed,), -9, dtype=torch.int32, device="cuda"),
            torch.full((8,), -9, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("name", ["deepseek_v3_small", "skewed_small", "mixtral_small", "deepseek_v3_decode_small"])
def test_static_scratch_route_matches_workspace_route_twice(name):
    w = W.get(name)
    dev = W.device_inputs(w)
    cfg = H.cfg_for(w)
    weights = H.weights_for(dev)

    # the existing entry point, with a workspace the caller allocated
    ws = H.workspace(cfg, w.n)
    idx0, tw0, cnt0, dg0 = _outputs(w)
    moe.moe_route(cfg, w.n, dev["x"], weights, idx0, tw0, cnt0, dg0, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK

    for call in range(2):
        idx, tw, cnt, dg = _outputs(w)
        moe.moe_route_static_scratch(cfg, w.n, dev["x"], weights, idx, tw, cnt, dg)
        torch.cuda.synchronize()
        diag = H.diag_dict(dg)
        assert diag["status"] == moe.MOE_OK, (call, diag)
        assert torch.equal(idx, idx0), call
        assert torch.equal(cnt, cnt0), call
        np.testing.assert_allclose(tw.cpu().numpy(), tw0.cpu().numpy(), rtol=2e-4, atol=1e-6)
        assert diag["refined_tokens"] == H.diag_dict(dg0)["refined_tokens"]
        assert diag["overflowed"] == H.diag_dict(dg0)["overflowed"]


def _fits(cfg, n, x, weights, outs):
    """True when n tokens fit the array (the call runs), False when it is refused as too large."""
    idx, tw, cnt, dg = outs
    try:
        moe.moe_route_static_scratch(cfg, n, x, weights, idx, tw, cnt, dg)
    except moe.MoeError as e:
        assert e.status == moe.MOE_ERR_WORKSPACE
        return False
    return True


def test_static_scratch_at_the_largest_batch_it_holds():
    """The size check against the router's real footprint: capacity routing (logits, the full
    per-token ranking and the per-block counts) at the largest token count the array holds,
    found by bisection on the entry point's own answer, matches moe_route on a workspace, twice;
    one token more is refused."""
    w = W.get("skewed_small", n=40000)
    dev = W.device_inputs(w)
    cfg = H.cfg_for(w)
    weights = H.weights_for(dev)
    big = _outputs(w)
    lo, hi = 1, w.n
    assert _fits(cfg, lo, dev["x"], weights, big) and not _fits(cfg, hi, dev["x"], weights, big)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if _fits(cfg, mid, dev["x"], weights, big):
            lo = mid
        else:
            hi = mid
    torch.cuda.synchronize()
    n = lo
    assert n > 10000, n  # E = 64 with a capacity: about 390 bytes of scratch per token
    wn = W.get("skewed_small", n=n)
    x = dev["x"][:n]
    ws = H.workspace(cfg, n)
    idx0, tw0, cnt0, dg0 = _outputs(wn)
    moe.moe_route(cfg, n, x, weights, idx0, tw0, cnt0, dg0, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    for call in range(2):
        idx, tw, cnt, dg = _outputs(wn)
        moe.moe_route_static_scratch(cfg, n, x, weights, idx, tw, cnt, dg)
        torch.cuda.synchronize()
        assert H.diag_dict(dg)["status"] == moe.MOE_OK, call
        assert torch.equal(idx, idx0), call
        assert torch.equal(cnt, cnt0), call
        np.testing.assert_allclose(tw.cpu().numpy(), tw0.cpu().numpy(), rtol=2e-4, atol=1e-6)
        assert H.diag_dict(dg)["overflowed"] == H.diag_dict(dg0)["overflowed"] > 0
    assert not _fits(cfg, n + 1, dev["x"], weights, big)


def test_static_scratch_requires_diag():
    """Without diag the device status word would stay in the shared array, unreadable."""
    w = W.get("mixtral_small")
    dev = W.device_inputs(w)
    idx, tw, cnt, _ = _outputs(w)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route_static_scratch(H.cfg_for(w), w.n, dev["x"], H.weights_for(dev), idx, tw, cnt, None)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG


def test_static_scratch_rejects_sizes_beyond_the_array():
    w = W.get("deepseek_v3_prefill")  # 16384 tokens x 256 experts of fp32 logits > 8 MiB
    cfg = H.cfg_for(w)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    weights = moe.make_weights(dummy, dummy, dummy, dummy)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route_static_scratch(cfg, w.n, dummy, weights, dummy, dummy, None, None)
    assert e.value.status == moe.MOE_ERR_WORKSPACE
