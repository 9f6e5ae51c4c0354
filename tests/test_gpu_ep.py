"""Expert parallelism on the GPU: every rank of a group driven by one process on
one device (all exchange buffers local, the steps of all ranks in stream
order), against the fp64 oracle layer on the concatenated batch.

Checked per case: the rows each owner received equal the oracle's receive
layout bit for bit (a pure copy); routing indices equal the oracle's (near-ties
exempt); the layer output is within the dtype's tolerance of the oracle and of
the single-device layer on the same batch. Ranks with no tokens and owners
receiving no rows are included. The flag barrier of the one-rank-per-process
mode is checked without a second rank running: once with the peer's arrivals
planted in advance (every wait ends at once), once with a peer that never
arrives (the bounded wait runs out and MOE_ERR_TIMEOUT reaches the status
word, the context stays usable).
"""
import numpy as np
import pytest
import torch

import top_routing_expert_router_b200 as moe
from oracle import oracle as O
from synth import workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu

MATS = ("gate", "up", "down")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _splits(n, world, seed):
    """Uneven contiguous token chunks, the first rank empty when world > 1."""
    if world == 1:
        return [n]
    rng = np.random.default_rng(seed)
    cut = np.sort(rng.integers(0, n + 1, world - 2))
    sizes = np.diff(np.concatenate([[0], cut, [n]])).tolist()
    return [0] + [int(v) for v in sizes]


def _rank_weights(w, dev, q, world):
    """Router, bias and shared experts of the layer; only the owned experts' matrices."""
    Eq = w.n_routed // world
    sl = slice(q * Eq, (q + 1) * Eq)
    if w.dtype == "fp8":
        scales = {k: dev["w_%s_s" % k][sl] for k in MATS}
        if "ws_gate_q" in dev:
            scales.update({"ws_" + k: dev["ws_%s_s" % k] for k in MATS})
        return moe.make_weights(dev["w_r"], dev["w_gate_q"][sl], dev["w_up_q"][sl], dev["w_down_q"][sl],
                                dev.get("ws_gate_q"), dev.get("ws_up_q"), dev.get("ws_down_q"), dev.get("bias"),
                                scales=scales)
    return moe.make_weights(dev["w_r"], dev["w_gate"][sl], dev["w_up"][sl], dev["w_down"][sl], dev.get("ws_gate"),
                            dev.get("ws_up"), dev.get("ws_down"), dev.get("bias"))


def run_ep(w, dev, world, splits, recv_rows=None):
    cfg = H.cfg_for(w)
    x = dev["x"]
    recv_rows = recv_rows or moe.moe_ep_recv_rows_bound(cfg, world, splits)
    bufs = dict(recv_x=[torch.zeros((recv_rows, w.d_model), dtype=x.dtype, device="cuda") for _ in range(world)],
                recv_out=[torch.zeros((recv_rows, w.d_model), dtype=x.dtype, device="cuda") for _ in range(world)],
                counts=[torch.zeros((world, w.n_routed), dtype=torch.int32, device="cuda") for _ in range(world)])
    group = moe.make_ep_group(recv_rows, **bufs)
    first = np.concatenate([[0], np.cumsum(splits)])
    ranks = []
    for q in range(world):
        n = splits[q]
        r = dict(n=n, x=x[first[q]:first[q + 1]], weights=_rank_weights(w, dev, q, world),
                 y=torch.empty((n, w.d_model), dtype=x.dtype, device="cuda"),
                 topk_idx=torch.empty((n, w.top_k), dtype=torch.int32, device="cuda"),
                 ws=torch.empty(moe.moe_ep_workspace_size(cfg, world, n, recv_rows), dtype=torch.uint8,
                                device="cuda"))
        ranks.append(r)
    moe.moe_ep_layer_forward(cfg, group, 0, ranks)
    for r in ranks:
        st = moe.moe_sync_status(r["ws"])
        assert st == moe.MOE_OK, moe.moe_status_string(st)
    return ranks, bufs


def _oracle(w, host):
    if w.dtype == "fp8":
        w8 = {k: (host["w_%s_q" % k], host["w_%s_s" % k]) for k in MATS}
        ws8 = {k: (host["ws_%s_q" % k], host["ws_%s_s" % k]) for k in MATS} if "ws_gate_q" in host else None
        return O.layer_fp8(H.oracle_cfg(w), host["x"], host["w_r"], host.get("bias"), w8, ws8)
    return O.layer(H.oracle_cfg(w), host["x"], host["w_r"], host["w_gate"], host["w_up"], host["w_down"],
                   host.get("bias"), host.get("ws_gate"), host.get("ws_up"), host.get("ws_down"))


CASES = [("mixtral_small", 2), ("mixtral_small", 4), ("mixtral_small", 8), ("deepseek_v2_small", 4),
         ("deepseek_v2_small", 8), ("deepseek_v3_small", 8), ("deepseek_v4_small", 2), ("ragged_small", 1),
         ("tiny_f32", 2), ("fp8_ragged_small", 2), ("fp8_ragged_small", 4), ("deepseek_v3_small_fp8", 8),
         # FP8 short tiles (received rows average at most 16 per owned expert); the second has
         # experts with more than 32 rows, so their groups span several short tiles
         ("deepseek_v3_decode_small_fp8", 8), ("fp8_skewed_small", 1)]


@pytest.mark.parametrize("name,world", CASES)
def test_ep_layer_matches_oracle(name, world):
    w = W.get(name)
    host, dev = W.host_inputs(w), W.device_inputs(w)
    splits = _splits(w.n, world, seed=world)
    ranks, bufs = run_ep(w, dev, world, splits)
    ref = _oracle(w, host)
    keep = ~ref["exempt"]
    idx = torch.cat([r["topk_idx"] for r in ranks]).cpu().numpy()
    np.testing.assert_array_equal(idx[keep], ref["topk_idx"][keep])
    y = torch.cat([r["y"] for r in ranks])
    tol = H.TOL["f32" if w.dtype == "f32" else "bf16"]
    assert H.rel_err(H.as_f64(y)[keep], ref["y"][keep]) <= tol
    # every owner received exactly the oracle's rows, in the oracle's order
    first = np.concatenate([[0], np.cumsum(splits)])
    lay = O.ep_recv_layout([ref["topk_idx"][first[q]:first[q + 1]] for q in range(world)], w.n_routed, world)
    xh = H.to_np(dev["x"])
    for q, (rows, _) in enumerate(lay):
        got = H.to_np(bufs["recv_x"][q][: len(rows)])
        np.testing.assert_array_equal(got, xh[first[rows[:, 0]] + rows[:, 1]])
    # same result as the single-device layer on the concatenated batch
    if w.dtype != "fp8":
        single = H.run_layer(w, dev)
        assert torch.equal(single["topk_idx"], torch.from_numpy(idx).cuda())
        assert H.rel_err(H.as_f64(y), H.as_f64(single["y"])) <= tol


def test_ep_v3_group_limit_bounds_the_ranks_a_token_reaches():
    """One expert group per rank: a token's experts lie on at most topk_group ranks."""
    w = W.get("deepseek_v3_small")
    dev = W.device_inputs(w)
    ranks, _ = run_ep(w, dev, 8, _splits(w.n, 8, seed=3))
    idx = torch.cat([r["topk_idx"] for r in ranks]).cpu().numpy()
    owners = idx // (w.n_routed // 8)
    assert max(len(set(row)) for row in owners.tolist()) <= w.topk_group


def test_ep_rejects_capacity_and_bad_groups():
    w = W.get("mixtral_small")
    dev = W.device_inputs(w)
    cfg = H.cfg_for(w)
    cap = H.cfg_for(W.get("drop_small"))
    with pytest.raises(moe.MoeError):
        moe.moe_ep_workspace_size(cfg, 3, 16, 64)  # 8 experts over 3 ranks
    buf = [torch.zeros((64, w.d_model), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    cnt = [torch.zeros((2, 16), dtype=torch.int32, device="cuda") for _ in range(2)]
    g = moe.make_ep_group(64, buf, buf, cnt)
    r = [dict(n=0, x=None, weights=H.weights_for(dev), y=None, ws=torch.empty(1 << 20, dtype=torch.uint8,
                                                                                 device="cuda"))]
    with pytest.raises(moe.MoeError) as e:
        moe.moe_ep_layer_forward(cap, g, 0, r * 2)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
    with pytest.raises(moe.MoeError) as e:  # 3 ranks of a 2-rank group
        moe.moe_ep_layer_forward(cfg, g, 0, r * 3)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as e:  # one rank per process needs the flag words
        moe.moe_ep_layer_forward(cfg, g, 1, r)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG


def _solo_rank0(w, dev, flags, recv_rows=2048):
    """Rank 0 of a two-rank group run alone (rank 1's buffers are local stand-ins nobody serves)."""
    cfg = H.cfg_for(w)
    world, n = 2, 128
    bufs = dict(recv_x=[torch.zeros((recv_rows, w.d_model), dtype=torch.bfloat16, device="cuda") for _ in range(2)],
                recv_out=[torch.zeros((recv_rows, w.d_model), dtype=torch.bfloat16, device="cuda") for _ in range(2)],
                counts=[torch.zeros((world, w.n_routed), dtype=torch.int32, device="cuda") for _ in range(2)])
    g = moe.make_ep_group(recv_rows, flags=flags, **bufs)
    ws = torch.empty(moe.moe_ep_workspace_size(cfg, world, n, recv_rows), dtype=torch.uint8, device="cuda")
    r = dict(n=n, x=dev["x"][:n], weights=_rank_weights(w, dev, 0, world),
             y=torch.empty((n, w.d_model), dtype=torch.bfloat16, device="cuda"), ws=ws)
    moe.moe_ep_layer_forward(cfg, g, 0, [r])
    return moe.moe_sync_status(ws)


def test_ep_barrier_passes_when_the_peer_has_arrived(monkeypatch):
    monkeypatch.setenv("MOE_EP_TIMEOUT_MS", "2000")
    w = W.get("mixtral_small")
    dev = W.device_inputs(w)
    flags = [torch.zeros(3, dtype=torch.int32, device="cuda") for _ in range(2)]
    flags[0][1] = 4  # rank 1's arrival at all four barriers of the call, planted in advance
    assert _solo_rank0(w, dev, flags) == moe.MOE_OK
    torch.cuda.synchronize()
    assert flags[0].tolist() == [4, 4, 4]  # own arrival, the peer's, the epoch counter
    assert flags[1].tolist() == [4, 0, 0]  # rank 0's arrival written into rank 1's words


def test_ep_barrier_times_out_when_the_peer_never_arrives(monkeypatch):
    monkeypatch.setenv("MOE_EP_TIMEOUT_MS", "100")
    w = W.get("mixtral_small")
    dev = W.device_inputs(w)
    flags = [torch.zeros(3, dtype=torch.int32, device="cuda") for _ in range(2)]
    assert _solo_rank0(w, dev, flags) == moe.MOE_ERR_TIMEOUT
    torch.cuda.synchronize()
    assert flags[0][2].item() == 4  # every barrier of the call still ran (without waiting after the first)
    # the context is still usable
    out = H.run_layer(w, dev)
    assert torch.isfinite(out["y"].float()).all()
