"""FP8 experts on the GPU (MOE_FP8) against the fp64 oracle.

Page "15. DeepSeek: MLA, MoE and MTP", FP8 section: E4M3 matrix inputs, one
UE8M0 scale per 1 x 128 activation tile and per 128 x 128 weight block. The
activation quantiser must match the oracle's codes and scale bytes exactly
(identical bf16 inputs, one correctly rounded conversion). Expert outputs and
layer outputs use the bf16 tolerance; both sides decide the E4M3 codes of h on
h held in bf16 (the kernel's binary32 sum rounded to bf16, the oracle's
binary64 sum rounded through binary32 to bf16), so codes differ only where the
two sums round to different bf16 values.
"""
import numpy as np
import pytest
import torch

import top_routing_expert_router_b200 as moe
from oracle import oracle as O
from synth import workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu

# fp8_ragged_small: 75 rows per expert (128 x 128 tiles); the others average at most 16 rows per
# expert, where the GEMM takes 32-row tiles (fp8_skewed_small: a Zipf-skewed router sends some
# experts more than 32 rows, so their groups span several short tiles).
FP8_SMALL = ["fp8_ragged_small", "deepseek_v3_small_fp8", "deepseek_v3_decode_small_fp8", "fp8_skewed_small"]
MATS = ("gate", "up", "down")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _weights(dev):
    scales = {k: dev["w_%s_s" % k] for k in MATS}
    if "ws_gate_q" in dev:
        scales.update({"ws_" + k: dev["ws_%s_s" % k] for k in MATS})
    return moe.make_weights(dev["w_r"], dev["w_gate_q"], dev["w_up_q"], dev["w_down_q"], dev.get("ws_gate_q"),
                            dev.get("ws_up_q"), dev.get("ws_down_q"), dev.get("bias"), scales=scales)


def _oracle_w8(host):
    w8 = {k: (host["w_%s_q" % k], host["w_%s_s" % k]) for k in MATS}
    ws8 = {k: (host["ws_%s_q" % k], host["ws_%s_s" % k]) for k in MATS} if "ws_gate_q" in host else None
    return w8, ws8


def _bf16_dev(a_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a_u16.view(np.int16)).cuda().view(torch.bfloat16)


def test_quantize_fp8_matches_oracle_bit_for_bit():
    w = W.get("fp8_ragged_small")
    x = W.host_inputs(w, names=["x"])["x"].copy()
    # magnitudes across many binades, exact in bf16 (power-of-two rescaling), and an all-zero row
    f = O.bf16_to_f64(x) * np.ldexp(1.0, np.arange(x.shape[0]) % 41 - 20)[:, None]
    f[7] = 0.0
    x = ((f.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
    codes = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    sb = torch.empty((x.shape[0], x.shape[1] // 128), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_fp8(_bf16_dev(x), codes, sb)
    torch.cuda.synchronize()
    rq, rs = O.quantize_rows(x)
    np.testing.assert_array_equal(sb.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rq)


def test_quantize_fp8_rejects_bad_shapes():
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((4, 100), dtype=torch.uint8, device="cuda")
    s = torch.empty((4, 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_quantize_fp8(x, q, s)


@pytest.mark.parametrize("bn", ["rule", "128", "256", "pair", "s128", "s256"])
@pytest.mark.parametrize("unit_scales", [False, True])
@pytest.mark.parametrize("name", FP8_SMALL)
def test_fp8_expert_ffn_parity(name, unit_scales, bn, monkeypatch):
    """Every tile shape matches the oracle: the one the rows per expert choose, one-SM 128-row tiles
    forced at both widths (128 x 128 with two accumulators, 128 x 256 with one), SM-pair 256 x 256
    tiles, and short 32-row tiles at both widths where the rows per expert allow them."""
    if bn == "rule":
        monkeypatch.delenv("MOE_FP8_BN", raising=False)
    else:
        monkeypatch.setenv("MOE_FP8_BN", bn)
    w = W.get(name)
    host, dev = W.host_inputs(w), W.device_inputs(w)
    if unit_scales:  # every weight block scale 2^0: isolates the activation-side scales
        for k in MATS:
            host["w_%s_s" % k][...] = 127
            dev["w_%s_s" % k].fill_(127)
    lg = O.router_logits(host["x"], host["w_r"])
    oi, _, _, _ = O.route_capacity(H.oracle_cfg(w), lg, host.get("bias"))
    counts, offsets, perm, dest = O.dispatch(oi, w.n_routed)
    xp_host = host["x"][perm]
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    eo = torch.empty((w.n * w.top_k, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, w.n, _bf16_dev(xp_host), torch.from_numpy(offsets).cuda(), _weights(dev), eo, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    got = H.as_f64(eo[: offsets[-1]])
    x64 = O.bf16_to_f64(xp_host)
    w8, _ = _oracle_w8(host)
    ref = np.zeros_like(got)
    for e in range(w.n_routed):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref[lo:hi] = O.swiglu_fp8(x64[lo:hi], *((w8[k][0][e], w8[k][1][e]) for k in MATS))
    assert H.rel_err(got, ref) <= H.TOL["bf16"]


@pytest.mark.parametrize("name", FP8_SMALL)
def test_fp8_layer_parity(name):
    w = W.get(name)
    host, dev = W.host_inputs(w), W.device_inputs(w)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    y = torch.empty((w.n, w.d_model), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(cfg, w.n, dev["x"], _weights(dev), y, ws, idx)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    w8, ws8 = _oracle_w8(host)
    r = O.layer_fp8(H.oracle_cfg(w), host["x"], host["w_r"], host.get("bias"), w8, ws8)
    keep = ~r["exempt"]
    np.testing.assert_array_equal(idx.cpu().numpy()[keep], r["topk_idx"][keep])
    assert H.rel_err(H.as_f64(y)[keep], r["y"][keep]) <= H.TOL["bf16"]


def test_fp8_config_rejects_dims_off_the_128_grid():
    w = W.get("fp8_ragged_small", d_model=200)
    cfg = H.cfg_for(w)
    with pytest.raises(moe.MoeError):
        moe.moe_workspace_size(cfg, w.n)
