"""Failure detection without a GPU fault.

Every barrier wait in the tensor-core GEMM is bounded. MOE_TEST_STALL=1 makes
each CTA's producer withhold its first copy, so the MMA's wait on that stage
can never complete; the kernel must give up after its (shortened) limit,
record MOE_ERR_TIMEOUT in the workspace status word, drain what is in flight,
release TMEM and return. The test reads the status on the host and then checks
that the same context still computes correct results.
"""
import numpy as np
import pytest
import torch

import top_routing_expert_router_b200 as moe
from oracle import oracle as O
from synth import workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.parametrize("mode", ["1sm", "2sm"])
def test_stalled_stage_reports_timeout_and_context_survives(mode, monkeypatch):
    monkeypatch.setenv("MOE_TC_MODE", mode)
    w = W.get("mixtral_small")
    host, dev = W.host_inputs(w), W.device_inputs(w)
    oi, _, _, _ = O.route_capacity(H.oracle_cfg(w), O.router_logits(host["x"], host["w_r"]))
    counts, offsets, perm, dest = O.dispatch(oi, w.n_routed)
    xp = torch.from_numpy(host["x"][perm].view(np.int16)).cuda().view(torch.bfloat16)
    offs = torch.from_numpy(offsets).cuda()
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    eo = torch.zeros((w.n * w.top_k, w.d_model), dtype=torch.bfloat16, device="cuda")

    monkeypatch.setenv("MOE_TEST_STALL", "1")
    moe.moe_expert_ffn(cfg, w.n, xp, offs, H.weights_for(dev), eo, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_ERR_TIMEOUT
    assert moe.moe_sync_status(ws) == moe.MOE_OK  # reading clears the word

    monkeypatch.delenv("MOE_TEST_STALL")
    moe.moe_expert_ffn(cfg, w.n, xp, offs, H.weights_for(dev), eo, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    got = H.as_f64(eo[: offsets[-1]])
    x64 = O.bf16_to_f64(host["x"][perm])
    ref = np.zeros_like(got)
    for e in range(w.n_routed):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref[lo:hi] = O.swiglu(x64[lo:hi], host["w_gate"][e], host["w_up"][e], host["w_down"][e])
    assert H.rel_err(got, ref) <= H.TOL[w.dtype]


def test_bf16_gemm_the_tensor_cores_cannot_take_is_unsupported(monkeypatch):
    """A bf16 layer never runs its matrix products on a slower path: when the tensor-core GEMM
    cannot take a shape (here forced by MOE_TEST_NO_TENSOR_MAPS=1, as if the driver had no tensor-map
    entry point) the call returns MOE_ERR_UNSUPPORTED. binary32 layers keep their CUDA-core GEMM."""
    w = W.get("mixtral_small")
    dev = W.device_inputs(w)
    monkeypatch.setenv("MOE_TEST_NO_TENSOR_MAPS", "1")
    with pytest.raises(moe.MoeError) as e:
        H.run_layer(w, dev)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
    wf = W.get("tiny_f32")
    out = H.run_layer(wf, W.device_inputs(wf))  # binary32: unaffected
    assert torch.isfinite(out["y"]).all()
    monkeypatch.delenv("MOE_TEST_NO_TENSOR_MAPS")
    out = H.run_layer(w, dev)
    assert torch.isfinite(out["y"]).all()


def test_router_with_expert_count_not_a_multiple_of_eight_runs_on_tensor_cores():
    """E = 5 experts in bf16: the binary32 logits rows are padded to a 16-byte stride and the
    last columns stored one by one, so the router GEMM stays on the tensor cores (and the
    indices still equal the oracle's)."""
    w = W.get("ragged_small")
    host, dev = W.host_inputs(w), W.device_inputs(w)
    out = H.run_layer(w, dev)
    oi, _, ex, _ = O.route_capacity(H.oracle_cfg(w), O.router_logits(host["x"], host["w_r"]), host.get("bias"))
    got = out["topk_idx"].cpu().numpy()
    assert (got[~ex] == oi[~ex]).all()
