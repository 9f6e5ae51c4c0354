"""Parity at the full workload sizes, in the configuration the benchmark runs.

Routing is checked on EVERY token: the GPU runs moe_layer_forward on the whole
batch and the oracle routes the whole batch from binary64 logits; expert
indices must be bit-exact on every token the oracle does not exempt (a
decision boundary closer than 1e-6 relative), gates within 2e-4 relative.
Under a capacity limit the comparison runs up to the first exempt token, since
the rule is sequential in token order. The dispatch of the GPU's indices
(offsets, stable permutation, slot destinations, permuted rows) is compared
with the oracle's counting sort on the whole batch, and the permutation is
checked to be a bijection between kept slots and permuted rows.

Layer outputs are checked on a sample of at least 64 tokens: the 32 whose
decisions are closest to a boundary in the oracle (the tokens the router has
to re-decide in binary64), the first and last token, and random ones. The
oracle recomputes those tokens expert by expert with the experts' weights
regenerated on the host.

Two router stress cases at d = 7168 scale the router weights 8x (sigmoid with
groups) and 4x (softmax) the recipe's scale, where the binary32 logit errors
are largest in absolute terms, and check every token's indices the same way.
FP8 layers at full size are checked on sampled tokens against the FP8 oracle.
"""
import numpy as np
import pytest
import torch

import top_routing_expert_router_b200 as moe
from oracle import oracle as O
from synth import workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu

FULL = ["tiny_f32", "mixtral_8x7b", "deepseek_v2", "deepseek_v3_prefill", "deepseek_v3_decode", "skewed_capacity"]
STRESS = ["deepseek_v3_route_x8", "softmax_7168_route_x4"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _router_inputs(w):
    return W.host_inputs(w, names=["x", "w_r"] + (["bias"] if w.bias_range else []))


def _decision_gap(w, logits, bias):
    """Per token, the smallest relative gap between two selection values whose order the routing
    depends on (group cut, adjacent kept experts, the k-th/(k+1)-th cut) in the oracle's binary64
    values. Used only to pick the hardest tokens for the output sample."""
    l = logits
    if w.score_fn == "softmax":
        v = l.copy()
    else:
        s = 1.0 / (1.0 + np.exp(-l)) if w.score_fn == "sigmoid" else np.sqrt(np.logaddexp(0.0, l))
        v = s + (bias.astype(np.float64) if bias is not None else 0.0)
    n, E = v.shape
    rel = lambda a, b: np.abs(a - b) / np.maximum(np.maximum(np.abs(a), np.abs(b)), 1e-300)
    gap = np.full(n, np.inf)
    elig = np.ones_like(v, bool)
    if w.n_group > 1:
        per = E // w.n_group
        vg = v.reshape(n, w.n_group, per)
        top2 = -np.sort(-vg, axis=2)[:, :, :2].sum(axis=2)
        order = np.argsort(-top2, axis=1, kind="stable")
        gs = np.take_along_axis(top2, order, axis=1)
        gap = np.minimum(gap, rel(gs[:, w.topk_group - 1], gs[:, w.topk_group]))
        keep = np.zeros((n, w.n_group), bool)
        np.put_along_axis(keep, order[:, : w.topk_group], True, axis=1)
        elig = np.repeat(keep, per, axis=1)
    ve = np.where(elig, v, -np.inf)
    srt = -np.sort(-ve, axis=1)[:, : w.top_k + 1]
    for j in range(min(w.top_k, srt.shape[1] - 1)):
        ok = np.isfinite(srt[:, j + 1])
        gap = np.where(ok, np.minimum(gap, rel(srt[:, j], srt[:, j + 1])), gap)
    return gap


def _sample(w, keep, gap, hard=32, rand=32):
    """Hardest non-exempt tokens by decision gap, plus the first, the last and random ones (every
    compared token when there are at most hard + rand of them)."""
    cand = np.nonzero(keep)[0]
    if len(cand) <= hard + rand:
        return cand.astype(np.int64)
    hardest = cand[np.argsort(gap[cand], kind="stable")[:hard]]
    rng = np.random.default_rng(0)
    pool = np.setdiff1d(cand, hardest)
    extra = rng.choice(pool, size=min(rand, len(pool)), replace=False) if len(pool) else []
    ends = [t for t in (0, w.n - 1) if keep[t]]
    return np.array(sorted({*hardest.tolist(), *np.asarray(extra).tolist(), *ends}), np.int64)


def _oracle_outputs(w, x_rows, idx, gates, fp8=False):
    """y of the sampled tokens from the oracle's routing, expert by expert (each expert's weights
    generated once), slots summed in order, then the shared experts."""
    d = w.d_model
    x64 = O.bf16_to_f64(x_rows) if x_rows.dtype == np.uint16 else x_rows.astype(np.float64)
    slot_out = np.zeros(idx.shape + (d,))
    for e in np.unique(idx[idx >= 0]):
        rows, slots = np.nonzero(idx == e)
        if fp8:
            mats = [(W.host_rows(w, f"w_{m}_q", [e])[0], W.host_rows(w, f"w_{m}_s", [e])[0]) for m in ("gate", "up", "down")]
            out = O.swiglu_fp8(x64[rows], *mats)
        else:
            wg, wu, wd = (W.host_rows(w, f"w_{m}", [e])[0] for m in ("gate", "up", "down"))
            out = O.swiglu(x64[rows], wg, wu, wd)
        slot_out[rows, slots] = out
    y = np.zeros((len(idx), d))
    for j in range(idx.shape[1]):
        y += np.where(idx[:, j : j + 1] >= 0, gates[:, j : j + 1], 0.0) * slot_out[:, j]
    if w.n_shared:
        if fp8:
            sh = W.host_inputs(w, names=[f"ws_{m}_{s}" for m in ("gate", "up", "down") for s in "qs"])
            y += O.swiglu_fp8(x64, *[(sh[f"ws_{m}_q"], sh[f"ws_{m}_s"]) for m in ("gate", "up", "down")])
        else:
            sh = W.host_inputs(w, names=["ws_gate", "ws_up", "ws_down"])
            y += O.swiglu(x64, sh["ws_gate"], sh["ws_up"], sh["ws_down"])
    return y


def _compare_routing(w, gi, gw, oi, ow, ex, st, diag):
    """Indices bit-exact on every token the comparison covers; returns that token mask."""
    if w.cap_policy != "none":
        stop = int(np.argmax(ex)) if ex.any() else w.n
        keep = np.arange(w.n) < stop
        if stop == w.n:
            assert diag["overflowed"] == st.overflowed and diag["dropped"] == st.dropped
    else:
        keep = ~ex
    bad = np.nonzero((gi[keep] != oi[keep]).any(axis=1))[0]
    assert bad.size == 0, (w.name, "index mismatches on non-exempt tokens:", np.nonzero(keep)[0][bad][:10])
    np.testing.assert_allclose(gw[keep], ow[keep], rtol=2e-4, atol=1e-6)
    return keep


def _check_dispatch(w, cfg, dev_x, gi_dev, gi):
    """moe_permute of the GPU's indices against the oracle's counting sort, whole batch."""
    n, k = w.n, w.top_k
    ws = H.workspace(cfg, n)
    offs = torch.empty(w.n_routed + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((n * k,), -7, dtype=torch.int32, device="cuda")
    dest = torch.empty((n, k), dtype=torch.int32, device="cuda")
    xp = torch.empty((n * k, w.d_model), dtype=dev_x.dtype, device="cuda")
    moe.moe_permute(cfg, n, dev_x, gi_dev, offs, perm, dest, xp, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    counts, offsets, operm, odest = O.dispatch(gi, w.n_routed)
    np.testing.assert_array_equal(offs.cpu().numpy(), offsets)
    kept = int(offsets[-1])
    gp = perm.cpu().numpy()[:kept]
    gd = dest.cpu().numpy()
    np.testing.assert_array_equal(gp, operm)
    np.testing.assert_array_equal(gd, odest)
    # bijection: every kept slot has its own row, that row holds the slot's token, dropped slots none
    kept_mask = gi >= 0
    rows = gd[kept_mask]
    assert (gd[~kept_mask] == -1).all()
    assert np.array_equal(np.sort(rows), np.arange(kept))
    tok = np.repeat(np.arange(n), k).reshape(n, k)[kept_mask]
    assert np.array_equal(gp[rows], tok)
    # the permuted rows are the tokens' rows, on the device
    src = dev_x.index_select(0, perm[:kept].long())
    assert torch.equal(xp[:kept].view(torch.int16) if xp.dtype == torch.bfloat16 else xp[:kept],
                       src.view(torch.int16) if src.dtype == torch.bfloat16 else src)


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(name):
    w = W.get(name)
    dev = W.device_inputs(w)
    got = H.run_layer(w, dev)
    gi = got["topk_idx"].cpu().numpy()
    gw = got["topk_w"].cpu().numpy()
    counts = got["counts"].cpu().numpy()
    diag = H.diag_dict(got["diag"])
    # whole-batch properties
    np.testing.assert_array_equal(counts, np.bincount(gi[gi >= 0], minlength=w.n_routed))
    assert counts.sum() == w.n * w.top_k - diag["dropped"]
    for row in gi:
        kept = row[row >= 0]
        assert len(set(kept.tolist())) == len(kept)
    # routing of every token against the oracle
    host = _router_inputs(w)
    bias = host.get("bias")
    lg = O.router_logits(host["x"], host["w_r"])
    oi, ow, ex, st = O.route_capacity(H.oracle_cfg(w), lg, bias)
    keep = _compare_routing(w, gi, gw, oi, ow, ex, st, diag)
    print(f"{name}: {int(keep.sum())} of {w.n} tokens compared, {int(ex.sum())} exempt, "
          f"refined_tokens {diag['refined_tokens']}, refined_logits {diag['refined_logits']}")
    # dispatch of the whole batch
    _check_dispatch(w, H.cfg_for(w), dev["x"], got["topk_idx"], gi)
    # outputs of the sampled tokens
    samples = _sample(w, keep, _decision_gap(w, lg, bias))
    assert len(samples) >= min(64, int(keep.sum()))
    ref = _oracle_outputs(w, host["x"][samples], oi[samples], ow[samples])
    y = H.as_f64(got["y"][torch.from_numpy(samples).cuda()])
    assert H.rel_err(y, ref) <= H.TOL[w.dtype], name


@pytest.mark.parametrize("name", STRESS)
def test_router_stress_every_token(name):
    """Router weights 4-8x the recipe's scale at d = 7168: every non-exempt token's indices equal
    the binary64 definition (the binary32 logits are certified or re-decided in binary64)."""
    w = W.get(name)
    dev = W.device_inputs(w, names=["x", "w_r"] + (["bias"] if w.bias_range else []))
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((w.n, w.top_k), dtype=torch.float32, device="cuda")
    cnt = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    dg = torch.zeros(8, dtype=torch.int32, device="cuda")
    wts = moe.make_weights(dev["w_r"], dev["w_r"], dev["w_r"], dev["w_r"], bias=dev.get("bias"))
    moe.moe_route(cfg, w.n, dev["x"], wts, idx, tw, cnt, dg, ws)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    host = _router_inputs(w)
    lg = O.router_logits(host["x"], host["w_r"])
    oi, ow, ex, st = O.route_capacity(H.oracle_cfg(w), lg, host.get("bias"))
    diag = H.diag_dict(dg)
    keep = _compare_routing(w, idx.cpu().numpy(), tw.cpu().numpy(), oi, ow, ex, st, diag)
    print(f"{name}: max|logit| {np.abs(lg).max():.1f}, {int(ex.sum())} exempt, "
          f"refined_tokens {diag['refined_tokens']}, refined_logits {diag['refined_logits']}")
    assert keep.mean() > 0.95


def _fp8_weights(dev):
    mats = ("gate", "up", "down")
    scales = {k: dev["w_%s_s" % k] for k in mats}
    scales.update({"ws_" + k: dev["ws_%s_s" % k] for k in mats if "ws_%s_s" % k in dev})
    return moe.make_weights(dev["w_r"], dev["w_gate_q"], dev["w_up_q"], dev["w_down_q"], dev.get("ws_gate_q"),
                            dev.get("ws_up_q"), dev.get("ws_down_q"), dev.get("bias"), scales=scales)


@pytest.mark.parametrize("name", ["deepseek_v3_prefill_fp8", "deepseek_v3_decode_fp8"])
def test_full_size_fp8_layer_sampled(name):
    """FP8 experts at the full V3 shapes: routing (bf16 router) of the sampled tokens bit-exact, and
    their outputs within the bf16 tolerance of the FP8 oracle (E4M3 activations in 1 x 128 tiles,
    UE8M0 128 x 128 weight blocks, binary64 products of the dequantised values)."""
    w = W.get(name)
    dev = W.device_inputs(w)
    cfg = H.cfg_for(w)
    ws = H.workspace(cfg, w.n)
    y = torch.empty((w.n, w.d_model), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((w.n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((w.n, w.top_k), dtype=torch.float32, device="cuda")
    moe.moe_layer_forward(cfg, w.n, dev["x"], _fp8_weights(dev), y, ws, idx, tw)
    assert moe.moe_sync_status(ws) == moe.MOE_OK
    rng = np.random.default_rng(1)
    samples = np.array(sorted({0, w.n - 1, *rng.choice(w.n, size=min(w.n, 30), replace=False).tolist()}))
    host = W.host_inputs(w, names=["w_r", "bias"])
    xs = W.host_rows(w, "x", samples)
    oi, ow, ex, _, _ = O.route(H.oracle_cfg(w), O.router_logits(xs, host["w_r"]), host["bias"])
    keep = ~ex
    gi = idx.cpu().numpy()[samples]
    np.testing.assert_array_equal(gi[keep], oi[keep])
    ref = _oracle_outputs(w, xs[keep], oi[keep], ow[keep], fp8=True)
    got = H.as_f64(y[torch.from_numpy(samples[keep]).cuda()])
    assert H.rel_err(got, ref) <= H.TOL["bf16"], name
