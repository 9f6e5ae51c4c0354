"""DeepSeek-V4-style routing on the GPU against the oracle: hash routing through
a token-id table (the router only weights the chosen experts) and the
auxiliary-loss-free bias update. sqrtsoftplus top-k routing itself is covered
by the deepseek_v4_small workload in test_gpu_parity.py."""
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


def _table(E, k, vocab, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(vocab)]).astype(np.int32)


def test_hash_routing_and_layer_match_oracle():
    w = W.get("deepseek_v4_small")
    dev, host = W.device_inputs(w), W.host_inputs(w)
    vocab = 97
    table = _table(w.n_routed, w.top_k, vocab, 5)
    tok = np.random.default_rng(6).integers(0, vocab, w.n).astype(np.int32)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((w.n, w.top_k), dtype=torch.float32, device="cuda")
    counts = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    weights = H.weights_for(dev)
    moe.moe_route_hash(cfg, w.n, dev["x"], torch.from_numpy(tok).cuda(), torch.from_numpy(table).cuda(), vocab,
                       weights, idx, tw, counts, None, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    ocfg = H.oracle_cfg(w)
    oi, ow = O.route_hash(ocfg, O.router_logits(host["x"], host["w_r"]), tok, table)
    np.testing.assert_array_equal(idx.cpu().numpy(), oi)
    np.testing.assert_allclose(tw.cpu().numpy(), ow, rtol=2e-4, atol=1e-6)
    np.testing.assert_array_equal(counts.cpu().numpy(), np.bincount(oi.ravel(), minlength=w.n_routed))
    # the rest of the layer through the staged entry points
    nk = w.n * w.top_k
    offs = torch.empty(w.n_routed + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(nk, dtype=torch.int32, device="cuda")
    dest = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    xp = torch.empty((nk, w.d_model), dtype=torch.bfloat16, device="cuda")
    eo = torch.empty_like(xp)
    y = torch.empty((w.n, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(cfg, w.n, dev["x"], idx, offs, perm, dest, xp, ws)
    moe.moe_expert_ffn(cfg, w.n, xp, offs, weights, eo, ws)
    moe.moe_combine(cfg, w.n, eo, dest, tw, dev["x"], weights, y, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    c2, off2, perm2, dest2 = O.dispatch(oi, w.n_routed)
    x64 = O.bf16_to_f64(host["x"])
    eo_ref = np.zeros((len(perm2), w.d_model))
    for e in range(w.n_routed):
        lo, hi = off2[e], off2[e + 1]
        if hi > lo:
            eo_ref[lo:hi] = O.swiglu(x64[perm2[lo:hi]], host["w_gate"][e], host["w_up"][e], host["w_down"][e])
    sh = O.swiglu(x64, host["ws_gate"], host["ws_up"], host["ws_down"])
    ref = O.combine(eo_ref, dest2, ow, sh)
    assert H.rel_err(H.as_f64(y), ref) <= H.TOL[w.dtype]


def test_hash_routing_rejects_out_of_range_ids_on_device():
    w = W.get("deepseek_v4_small", n=8)
    dev = W.device_inputs(w)
    vocab = 10
    table = _table(w.n_routed, w.top_k, vocab, 7)
    tok = np.array([0, 1, 2, 3, 99, 5, -1, 9], np.int32)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((w.n, w.top_k), dtype=torch.float32, device="cuda")
    moe.moe_route_hash(cfg, w.n, dev["x"], torch.from_numpy(tok).cuda(), torch.from_numpy(table).cuda(), vocab,
                       H.weights_for(dev), idx, tw, None, None, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_ERR_INVALID_ARG
    gi = idx.cpu().numpy()
    assert (gi[4] == -1).all() and (gi[6] == -1).all() and (tw.cpu().numpy()[4] == 0).all()
    np.testing.assert_array_equal(gi[[0, 1, 2, 3, 5, 7]], table[tok[[0, 1, 2, 3, 5, 7]]])


def test_bias_update_matches_oracle_bit_for_bit():
    w = W.get("deepseek_v3_small")
    dev = W.device_inputs(w)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((w.n, w.top_k), dtype=torch.float32, device="cuda")
    counts = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_route(cfg, w.n, dev["x"], H.weights_for(dev), idx, tw, counts, None, ws)
    bias0 = dev["bias"].cpu().numpy().copy()
    moe.moe_bias_update(cfg, counts, dev["bias"], 0.001)
    torch.cuda.synchronize()
    ref = O.bias_update(counts.cpu().numpy(), bias0, float(np.float32(0.001)))
    np.testing.assert_array_equal(dev["bias"].cpu().numpy(), ref.astype(np.float32))
    assert (dev["bias"].cpu().numpy() != bias0).any()
