"""Parity of the CUDA path (called through the C ABI) with the fp64 CPU oracle.

Indices, permutations and counts must be bit-exact, except for tokens the
oracle marks exempt (a decision boundary closer than 1e-6 relative); the
tie-stress workloads have exact integer logits and must match on every token.
Layer outputs must satisfy max_i |y_i - r_i| / max(|r_i|, rms(r)) <= 2e-2 (bf16)
or 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

import top_routing_expert_router_b200 as moe
from oracle import oracle as O
from synth import synth, workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu

SMALL = ["tiny_f32", "mixtral_small", "deepseek_v2_small", "deepseek_v3_small", "deepseek_v3_decode_small",
         "skewed_small", "drop_small", "ragged_small", "deepseek_v4_small", "tie_softmax", "tie_sigmoid"]


def _tile_mode(mode, monkeypatch):
    """1sm: one-SM 128-row tiles; 2sm: SM-pair 256 x 256 tiles; 2sm_wide: SM-pair 256 x 512 tiles
    (the default mix, wide gate/up tiles for small groups, runs in every other test)."""
    monkeypatch.setenv("MOE_TC_MODE", "1sm" if mode == "1sm" else "2sm")
    monkeypatch.setenv("MOE_TC_WIDE", "1" if mode == "2sm_wide" else "0")


TILE_MODES = ["1sm", "2sm", "2sm_wide"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _oracle_route(w, host):
    lg = O.router_logits(host["x"], host["w_r"])
    return O.route_capacity(H.oracle_cfg(w), lg, host.get("bias"))


@pytest.mark.parametrize("name", ["mixtral_small", "deepseek_v3_small", "tiny_f32", "skewed_small"])
def test_device_inputs_equal_host_inputs(name):
    w = W.get(name)
    dev = W.device_inputs(w)
    host = W.host_inputs(w)
    for k in host:
        assert (H.to_np(dev[k]) == host[k]).all(), k


@pytest.mark.parametrize("name", SMALL)
def test_route_parity(name, w=None):
    w = w or W.get(name)
    _check_route(w, W.device_inputs(w), W.host_inputs(w))


def _check_route(w, dev, host):
    """moe_route on the device inputs against the oracle's routing of the host inputs; returns the
    diagnostics."""
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((w.n, w.top_k), dtype=torch.float32, device="cuda")
    counts = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    dg = torch.zeros(8, dtype=torch.int32, device="cuda")
    moe.moe_route(cfg, w.n, dev["x"], H.weights_for(dev), idx, tw, counts, dg, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    oi, ow, ex, st = _oracle_route(w, host)
    gi, gw = idx.cpu().numpy(), tw.cpu().numpy()
    diag = H.diag_dict(dg)
    if w.ternary:
        ex = np.zeros_like(ex)  # exact integer logits: every token must match, ties included
        assert diag["refined_tokens"] > 0
    if w.cap_policy != "none":
        # a near-tie can cascade through the capacity counts: compare up to the first exempt token
        stop = int(np.argmax(ex)) if ex.any() else w.n
        np.testing.assert_array_equal(gi[:stop], oi[:stop])
        if stop == w.n:
            assert diag["overflowed"] == st.overflowed and diag["dropped"] == st.dropped
        keep = np.arange(w.n) < stop
    else:
        keep = ~ex
        np.testing.assert_array_equal(gi[keep], oi[keep])
    np.testing.assert_allclose(gw[keep], ow[keep], rtol=2e-4, atol=1e-6)
    if keep.all():
        np.testing.assert_array_equal(counts.cpu().numpy(), np.bincount(oi[oi >= 0], minlength=w.n_routed))
        assert diag["max_load"] == np.bincount(oi[oi >= 0], minlength=w.n_routed).max()
    assert ex.mean() < 0.05
    return diag


@pytest.mark.parametrize("name,n,refines", [("deepseek_v3_small", 333, True), ("deepseek_v3_small", 3000, True),
                                            ("mixtral_small", 700, False), ("skewed_small", 2000, True)])
def test_route_parity_with_subnormal_token_values(name, n, refines):
    """Every token's row holds bf16 subnormals and a zero next to its normal values. The routing
    must still equal the oracle's, which takes the exact binary64 values of the same inputs,
    including for the tokens the binary64 refinement re-decides. From 2048 tokens the one-pass
    router queues the uncertain tokens for that refinement. The Mixtral-shaped case certifies
    every token in binary32."""
    w = W.get(name, n=n)
    dev, host = W.device_inputs(w), W.host_inputs(w)
    x = host["x"].copy()
    assert x.dtype == np.uint16
    x[:, 0] = 0x0001  # smallest positive subnormal, 2^-133
    x[:, 1] = 0x807F  # largest negative subnormal
    x[:, 2] = 0x0000
    dev = dict(dev, x=torch.from_numpy(x.view(np.int16)).to("cuda").view(torch.bfloat16))
    host = dict(host, x=x)
    diag = _check_route(w, dev, host)
    if refines:
        assert diag["refined_tokens"] > 0  # the refinement ran on rows holding subnormals


@pytest.mark.parametrize("policy", ["overflow_next", "drop"])
@pytest.mark.parametrize("k", [1, 3, 4, 6, 8])
def test_capacity_route_parity_across_top_k(k, policy):
    """The capacity kernel keeps a token's choices in registers for top_k 1, 2, 4, 8 and in a
    local array otherwise; both match the oracle's greedy."""
    w = W.get("skewed_small", top_k=k, cap_policy=policy, n=1500)
    test_route_parity(w.name, w)


# From 2048 tokens the router decides in the tensor-core epilogue (one pass) and re-decides only
# the uncertain tokens in binary64; the tie workloads send many tokens down that second path.
ONE_PASS = ["mixtral_small", "deepseek_v2_small", "deepseek_v3_small", "deepseek_v4_small", "ragged_small",
            "tie_softmax", "tie_sigmoid"]


@pytest.mark.parametrize("name", ONE_PASS)
def test_one_pass_route_parity(name):
    w = W.get(name, n=2304 if name != "ragged_small" else 4100)
    test_route_parity(w.name, w)


@pytest.mark.parametrize("mode", ["grid", "1cta"])
@pytest.mark.parametrize("policy", ["overflow_next", "drop"])
@pytest.mark.parametrize("k", [1, 2, 3, 8])
def test_capacity_on_many_ctas(k, policy, mode, monkeypatch):
    """20 000 tokens: the capacity rule on a cooperative grid of 20 CTAs (one fill event per round)
    and on the one-CTA kernel, both against the oracle's sequential greedy."""
    if mode == "1cta":
        monkeypatch.setenv("MOE_CAP_MODE", "1cta")
    w = W.get("skewed_small", top_k=k, cap_policy=policy, n=20000)
    test_route_parity(w.name, w)


@pytest.mark.parametrize("policy", ["overflow_next", "drop"])
@pytest.mark.parametrize("E", [8, 24, 40, 100, 128])
def test_capacity_grid_expert_counts(E, policy):
    """6000 tokens on 6 CTAs of the chained grid, across the expert counts its staging and walks
    distinguish: whole rankings of at most 64 experts with the position masks (E a multiple of 8),
    rankings staged token by token (E = 100), and walks that go on in global memory past the 64
    staged entries (E = 128)."""
    w = W.get("skewed_small", n_routed=E, top_k=2, cap_policy=policy, n=6000)
    test_route_parity(w.name, w)


@pytest.mark.parametrize("name", ["mixtral_small", "deepseek_v2_small", "skewed_small", "drop_small", "tiny_f32"])
def test_permute_parity(name):
    w = W.get(name)
    host = W.host_inputs(w, names=["x", "w_r", "bias"] if w.bias_range else ["x", "w_r"])
    oi, _, _, _ = _oracle_route(w, host)
    counts, offsets, perm, dest = O.dispatch(oi, w.n_routed)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    x = W.device_inputs(w, names=["x"])["x"]
    nk = w.n * w.top_k
    g_off = torch.empty(w.n_routed + 1, dtype=torch.int32, device="cuda")
    g_perm = torch.full((nk,), -7, dtype=torch.int32, device="cuda")
    g_dest = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    g_xp = torch.empty((nk, w.d_model), dtype=x.dtype, device="cuda")
    moe.moe_permute(cfg, w.n, x, torch.from_numpy(oi).cuda(), g_off, g_perm, g_dest, g_xp, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    np.testing.assert_array_equal(g_off.cpu().numpy(), offsets)
    kept = int(offsets[-1])
    np.testing.assert_array_equal(g_perm.cpu().numpy()[:kept], perm)
    np.testing.assert_array_equal(g_dest.cpu().numpy(), dest)
    assert (H.to_np(g_xp[:kept]) == host["x"][perm]).all()


@pytest.mark.parametrize("name", ["tiny_f32", "mixtral_small", "deepseek_v2_small", "deepseek_v3_small",
                                  "deepseek_v3_decode_small", "skewed_small", "ragged_small"])
def test_expert_ffn_parity(name):
    w = W.get(name)
    host = W.host_inputs(w)
    dev = W.device_inputs(w)
    oi, _, _, _ = _oracle_route(w, host)
    counts, offsets, perm, dest = O.dispatch(oi, w.n_routed)
    xp_host = host["x"][perm]
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    xp = torch.from_numpy(xp_host.view(np.int16) if xp_host.dtype == np.uint16 else xp_host).cuda()
    if w.dtype == "bf16":
        xp = xp.view(torch.bfloat16)
    eo = torch.empty((w.n * w.top_k, w.d_model), dtype=xp.dtype, device="cuda")
    moe.moe_expert_ffn(cfg, w.n, xp, torch.from_numpy(offsets).cuda(), H.weights_for(dev), eo, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    got = H.as_f64(eo[: offsets[-1]])
    x64 = O.bf16_to_f64(xp_host)
    ref = np.zeros_like(got)
    for e in range(w.n_routed):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref[lo:hi] = O.swiglu(x64[lo:hi], host["w_gate"][e], host["w_up"][e], host["w_down"][e])
    assert H.rel_err(got, ref) <= H.TOL[w.dtype]


@pytest.mark.parametrize("name", ["tiny_f32", "deepseek_v2_small", "deepseek_v3_small"])
def test_combine_parity(name):
    w = W.get(name)
    host = W.host_inputs(w)
    dev = W.device_inputs(w)
    oi, ow, _, _ = _oracle_route(w, host)
    counts, offsets, perm, dest = O.dispatch(oi, w.n_routed)
    rows = int(offsets[-1])
    # synthetic expert outputs in the layer's dtype
    eo_host = synth.host((rows, w.d_model), w.dtype, 0, 77, synth.NORMAL, 1.0)
    eo = torch.from_numpy(eo_host.view(np.int16) if w.dtype == "bf16" else eo_host).cuda()
    if w.dtype == "bf16":
        eo = eo.view(torch.bfloat16)
    tw32 = ow.astype(np.float32)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    y = torch.empty((w.n, w.d_model), dtype=eo.dtype, device="cuda")
    moe.moe_combine(cfg, w.n, eo, torch.from_numpy(dest).cuda(), torch.from_numpy(tw32).cuda(), dev["x"],
                    H.weights_for(dev), y, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    sh = None
    if w.n_shared:
        sh = O.swiglu(O.bf16_to_f64(host["x"]), host["ws_gate"], host["ws_up"], host["ws_down"])
    ref = O.combine(O.bf16_to_f64(eo_host), dest, tw32.astype(np.float64), sh)
    assert H.rel_err(H.as_f64(y), ref) <= H.TOL[w.dtype]


@pytest.mark.parametrize("name", SMALL)
def test_layer_parity(name):
    w = W.get(name)
    dev, host = W.device_inputs(w), W.host_inputs(w)
    got = H.run_layer(w, dev)
    r = O.layer(H.oracle_cfg(w), host["x"], host["w_r"], host["w_gate"], host["w_up"], host["w_down"],
                host.get("bias"), host.get("ws_gate"), host.get("ws_up"), host.get("ws_down"))
    gi = got["topk_idx"].cpu().numpy()
    ex = r["exempt"] if not w.ternary else np.zeros(w.n, bool)
    if w.cap_policy != "none" and ex.any():
        keep = np.arange(w.n) < int(np.argmax(ex))
    else:
        keep = ~ex
    np.testing.assert_array_equal(gi[keep], r["topk_idx"][keep])
    y = H.as_f64(got["y"])
    assert H.rel_err(y[keep], r["y"][keep]) <= H.TOL[w.dtype]


def test_layer_is_deterministic():
    w = W.get("deepseek_v3_small")
    dev = W.device_inputs(w)
    a = H.run_layer(w, dev)["y"].clone()
    b = H.run_layer(w, dev)["y"]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_zero_tokens_is_a_noop():
    w = W.get("mixtral_small")
    dev = W.device_inputs(w)
    got = H.run_layer(w, dev, n=0)
    assert got["counts"].sum().item() == 0


def test_single_token_and_ragged_sizes():
    w = W.get("deepseek_v3_small")
    dev, host = W.device_inputs(w), W.host_inputs(w)
    for n in (1, 3, 129):
        got = H.run_layer(w, {k: (v[:n] if k == "x" else v) for k, v in dev.items()}, n=n)
        r = O.layer(H.oracle_cfg(w), host["x"][:n], host["w_r"], host["w_gate"], host["w_up"], host["w_down"],
                    host.get("bias"), host.get("ws_gate"), host.get("ws_up"), host.get("ws_down"))
        keep = ~r["exempt"]
        np.testing.assert_array_equal(got["topk_idx"].cpu().numpy()[keep], r["topk_idx"][keep])
        assert H.rel_err(H.as_f64(got["y"])[keep], r["y"][keep]) <= H.TOL[w.dtype]


def _staged_layer(w, dev):
    """The layer through the staged entry points: route, permute (permuted copy), expert FFN, combine."""
    n, k, d = w.n, w.top_k, w.d_model
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, n)
    wts = H.weights_for(dev)
    idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((n, k), dtype=torch.float32, device="cuda")
    counts = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    dg = torch.zeros(8, dtype=torch.int32, device="cuda")
    offs = torch.empty(w.n_routed + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(n * k, dtype=torch.int32, device="cuda")
    dest = torch.empty((n, k), dtype=torch.int32, device="cuda")
    xp = torch.empty((n * k, d), dtype=dev["x"].dtype, device="cuda")
    eo = torch.empty((n * k, d), dtype=dev["x"].dtype, device="cuda")
    y = torch.empty((n, d), dtype=dev["x"].dtype, device="cuda")
    moe.moe_route(cfg, n, dev["x"], wts, idx, tw, counts, dg, ws)
    moe.moe_permute(cfg, n, dev["x"], idx, offs, perm, dest, xp, ws)
    moe.moe_expert_ffn(cfg, n, xp, offs, wts, eo, ws)
    moe.moe_combine(cfg, n, eo, dest, tw, dev["x"], wts, y, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    return y


@pytest.mark.parametrize("mode", TILE_MODES)
@pytest.mark.parametrize("name", ["mixtral_small", "deepseek_v2_small", "deepseek_v3_small", "ragged_small"])
def test_layer_equals_staged_path(name, mode, monkeypatch):
    """moe_layer_forward (shared experts on the side stream) equals route -> permute ->
    expert FFN -> combine through the staged entry points bit for bit."""
    _tile_mode(mode, monkeypatch)
    w = W.get(name)
    dev = W.device_inputs(w)
    fused = H.run_layer(w, dev)["y"]
    assert torch.equal(fused, _staged_layer(w, dev))




# Group sizes around the 128-row and 256-row tile edges: empty groups, one row,
# exact multiples, one past them, and groups whose last tile is half height.
EDGE_COUNTS = [0, 1, 64, 127, 128, 129, 255, 256, 257, 300, 384, 385, 513, 640, 0]


@pytest.mark.parametrize("mode", TILE_MODES)
def test_expert_ffn_tile_edges(mode, monkeypatch):
    """Caller-given group offsets at every tile edge; d and I leave ragged n- and k-tiles."""
    _tile_mode(mode, monkeypatch)
    counts = np.array(EDGE_COUNTS, np.int32)
    rows = int(counts.sum())
    w = W.get("ragged_small", n=rows, d_model=320, n_routed=len(counts), top_k=1, moe_intermediate_size=200,
              n_shared=0, renormalize=False)
    host = W.host_inputs(w, names=["x", "w_gate", "w_up", "w_down"])
    dev = W.device_inputs(w, names=["x", "w_gate", "w_up", "w_down"])
    offsets = np.zeros(len(counts) + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, rows)
    eo = torch.empty((rows, w.d_model), dtype=dev["x"].dtype, device="cuda")
    wts = moe.make_weights(None, dev["w_gate"], dev["w_up"], dev["w_down"])
    moe.moe_expert_ffn(cfg, rows, dev["x"], torch.from_numpy(offsets).cuda(), wts, eo, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    got = H.as_f64(eo)
    x64 = O.bf16_to_f64(host["x"])
    for e in range(len(counts)):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref = O.swiglu(x64[lo:hi], host["w_gate"][e], host["w_up"][e], host["w_down"][e])
            assert H.rel_err(got[lo:hi], ref) <= H.TOL[w.dtype], (e, int(counts[e]))


@pytest.mark.parametrize("mode", TILE_MODES)
@pytest.mark.parametrize("name", ["mixtral_small", "deepseek_v3_small", "ragged_small", "deepseek_v2_small"])
def test_expert_ffn_both_tile_modes(name, mode, monkeypatch):
    """The 128-row single-SM tiles and the 256-row SM-pair tiles (256 and 512 wide) match the oracle."""
    _tile_mode(mode, monkeypatch)
    test_expert_ffn_parity(name)
    w = W.get(name)
    dev, host = W.device_inputs(w), W.host_inputs(w)
    got = H.run_layer(w, dev)
    r = O.layer(H.oracle_cfg(w), host["x"], host["w_r"], host["w_gate"], host["w_up"], host["w_down"],
                host.get("bias"), host.get("ws_gate"), host.get("ws_up"), host.get("ws_down"))
    keep = ~r["exempt"]
    assert H.rel_err(H.as_f64(got["y"])[keep], r["y"][keep]) <= H.TOL[w.dtype]
