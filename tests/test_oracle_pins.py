"""Pins of the fp64 CPU oracle to facts outside itself.

Each test ties one oracle function to something the oracle does not compute
itself: integers printed on the pages, hand-worked examples, a library routine
(numpy/torch/scipy) that solves a special case, brute-force enumeration, or a
closed form. A dropped term, a wrong sign or index, or a transposed operand in
the oracle fails at least one of these.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import oracle as O
from synth import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _cfg(E, k, **kw):
    base = dict(d_model=1, n_routed=E, top_k=k, moe_intermediate_size=1)
    base.update(kw)
    return O.Cfg(**base)


# ---------------------------------------------------------------- parameter ledger (printed integers)


def test_deepseek_v3_ledger_matches_printed_totals():
    g = _gold("deepseek_param_ledger.json")["deepseek_v3"]
    total, active = O.ds_params(**g["arch"])
    assert total == g["total"] == 671026404352
    assert active == g["active"] == 37552282624
    a = g["arch"]
    # per-module integers printed beside the totals
    assert 3 * a["d_model"] * a["moe_inter"] == g["per_expert"]
    assert 3 * a["d_model"] * a["dense_inter"] == g["dense_ffn"]
    assert a["n_routed"] * a["d_model"] == g["router"]
    assert a["vocab"] * a["d_model"] == g["embedding"]


def test_deepseek_v2_ledger_matches_printed_total():
    g = _gold("deepseek_param_ledger.json")["deepseek_v2"]
    total, active = O.ds_params(**g["arch"])
    assert total == g["total"] == 235741434880
    assert round(active / 1e9) == 21  # the page's "21B activated"


def test_ledger_mla_term():
    # With every non-MLA term zeroed except norms, total = layers * MLA + norms.
    g = _gold("deepseek_param_ledger.json")["deepseek_v3"]
    a = dict(g["arch"], first_k_dense=0, dense_inter=0, n_routed=0, n_shared=0, top_k=0, vocab=0)
    a["n_layers"] = 1
    total, _ = O.ds_params(**a)
    assert total - (2 * 7168 + 7168) == g["per_layer_mla"]


# ---------------------------------------------------------------- router logits


def test_router_logits_match_numpy_matmul():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((37, 53)).astype(np.float32)
    w = rng.standard_normal((11, 53)).astype(np.float32)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    np.testing.assert_allclose(O.router_logits(x, w), ref, rtol=1e-12, atol=1e-12)


def test_router_logits_bf16_inputs_widened_exactly():
    w = W.get("mixtral_small")
    inp = W.host_inputs(w, names=["x", "w_r"])
    ref = O.bf16_to_f64(inp["x"]) @ O.bf16_to_f64(inp["w_r"]).T
    np.testing.assert_allclose(O.router_logits(inp["x"], inp["w_r"]), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- selection: worked examples


@pytest.mark.parametrize("case", ["softmax_ties", "softmax_tie_at_cut"])
def test_softmax_worked_examples(case):
    g = _gold("routing_worked_examples.json")[case]
    lg = np.array(g["logits"])
    idx, w, ex, _, _ = O.route(_cfg(lg.shape[1], g["top_k"]), lg)
    assert idx.tolist() == g["expect_idx"]


def test_sigmoid_group_worked_example():
    g = _gold("routing_worked_examples.json")["sigmoid_groups"]
    lg = np.array(g["logits"])
    cfg = _cfg(8, g["top_k"], score_fn="sigmoid", n_group=g["n_group"], topk_group=g["topk_group"],
               renormalize=True, routed_scaling_factor=g["routed_scaling_factor"])
    idx, w, ex, _, _ = O.route(cfg, lg, bias=np.zeros(8, np.float32))
    assert idx.tolist() == g["expect_idx"]
    np.testing.assert_allclose(w, g["expect_w"], rtol=1e-15)


def test_sigmoid_bias_worked_example():
    g = _gold("routing_worked_examples.json")["sigmoid_bias_selection_only"]
    lg = np.array(g["logits"])
    b = np.array(g["bias"], np.float32)
    for renorm, key in ((True, "expect_w_renorm"), (False, "expect_w_raw")):
        cfg = _cfg(4, 1, score_fn="sigmoid", renormalize=renorm)
        idx, w, _, _, _ = O.route(cfg, lg, bias=b)
        assert idx.tolist() == g["expect_idx"]
        np.testing.assert_allclose(w, g[key], rtol=1e-15)


# ---------------------------------------------------------------- selection: library and brute force


def _lexsort_topk(vals, k):
    """Plain top-k by a library sort: descending value, ties to lower index."""
    E = vals.shape[1]
    out = []
    for row in vals:
        order = np.lexsort((np.arange(E), -row))
        out.append(order[:k])
    return np.array(out, np.int32)


def test_plain_topk_reduces_to_library_sort():
    rng = np.random.default_rng(2)
    lg = rng.standard_normal((200, 19))
    lg[:20] = np.round(lg[:20])  # exact ties
    idx, w, _, _, _ = O.route(_cfg(19, 5), lg)
    np.testing.assert_array_equal(idx, _lexsort_topk(lg, 5))
    p = scipy.special.softmax(lg, axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=1e-13)


def test_renormalised_softmax_gates_equal_softmax_of_selected_logits():
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((50, 8)) * 3
    idx, w, _, _, _ = O.route(_cfg(8, 2, renormalize=True), lg)
    sel = np.take_along_axis(lg, idx, 1)
    np.testing.assert_allclose(w, scipy.special.softmax(sel, axis=1), rtol=1e-13)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)


def _brute_group_topk(c, G, keep, k):
    """Enumerate group subsets, then expert subsets (lexicographically first among the best)."""
    E = len(c)
    per = E // G
    gscore = [max(c[g * per + a] + c[g * per + b] for a in range(per) for b in range(per) if a != b)
              for g in range(G)]
    best_groups = None
    for gs in itertools.combinations(range(G), keep):
        s = math.fsum(gscore[g] for g in gs)  # correctly rounded: order-independent
        if best_groups is None or s > best_groups[0]:
            best_groups = (s, gs)
    elig = [e for e in range(E) if e // per in best_groups[1]]
    best = None
    for es in itertools.combinations(elig, k):
        s = math.fsum(c[e] for e in es)
        if best is None or s > best[0]:
            best = (s, es)
    return sorted(best[1], key=lambda e: (-c[e], e))


@pytest.mark.parametrize("integer_logits", [False, True])
def test_group_limited_topk_matches_brute_force(integer_logits):
    rng = np.random.default_rng(4 + integer_logits)
    E, G, keep, k = 12, 4, 2, 3
    lg = rng.integers(-2, 3, (300, E)).astype(np.float64) if integer_logits else rng.standard_normal((300, E))
    bias = np.zeros(E, np.float32) if integer_logits else rng.uniform(-0.1, 0.1, E).astype(np.float32)
    cfg = _cfg(E, k, score_fn="sigmoid", n_group=G, topk_group=keep, renormalize=True,
               routed_scaling_factor=2.5)
    idx, w, ex, _, _ = O.route(cfg, lg, bias=bias)
    s = scipy.special.expit(lg)
    c = s + bias.astype(np.float64)
    for t in range(lg.shape[0]):
        assert idx[t].tolist() == _brute_group_topk(c[t], G, keep, k), t
    sel = np.take_along_axis(s, idx, 1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True) * 2.5, rtol=1e-13)
    if integer_logits:
        assert ex.any()  # exact ties are flagged


def test_group_invariants_on_v3_shapes():
    rng = np.random.default_rng(6)
    E, G, keep, k = 256, 8, 4, 8
    lg = rng.standard_normal((400, E))
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    cfg = _cfg(E, k, score_fn="sigmoid", n_group=G, topk_group=keep, renormalize=True,
               routed_scaling_factor=2.5)
    idx, w, _, _, _ = O.route(cfg, lg, bias=bias)
    c = scipy.special.expit(lg) + bias
    gs = np.sort(c.reshape(-1, G, E // G), axis=2)[:, :, -2:].sum(2)
    for t in range(lg.shape[0]):
        assert len(set(idx[t].tolist())) == k
        kept = set(np.lexsort((np.arange(G), -gs[t]))[:keep].tolist())
        assert all(e // (E // G) in kept for e in idx[t])
    np.testing.assert_allclose(w.sum(1), 2.5, rtol=1e-13)
    # a huge bias on one expert forces it (and its group) in
    b2 = bias.copy()
    b2[77] = 100.0
    idx2, _, _, _, _ = O.route(cfg, lg, bias=b2)
    assert (idx2[:, 0] == 77).all()


def test_bias_changes_selection_never_gate_values():
    rng = np.random.default_rng(7)
    E, k = 64, 6
    lg = rng.standard_normal((500, E))
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    cfg = _cfg(E, k, score_fn="sigmoid", n_group=8, topk_group=4, renormalize=True, routed_scaling_factor=2.5)
    i0, w0, _, _, _ = O.route(cfg, lg, bias=np.zeros(E, np.float32))
    i1, w1, _, _, _ = O.route(cfg, lg, bias=bias)
    same = (np.sort(i0, 1) == np.sort(i1, 1)).all(1)
    assert same.any() and (~same).any()
    for t in np.nonzero(same)[0]:
        a = dict(zip(i0[t], w0[t]))
        b = dict(zip(i1[t], w1[t]))
        assert a.keys() == b.keys()
        # same values up to the order of the normalising sum (slots may be reordered)
        np.testing.assert_allclose([a[e] for e in a], [b[e] for e in a], rtol=1e-15)
    # gates always use raw scores: w = s_sel / sum s_sel * rsf
    s = scipy.special.expit(lg)
    sel = np.take_along_axis(s, i1, 1)
    np.testing.assert_allclose(w1, sel / sel.sum(1, keepdims=True) * 2.5, rtol=1e-13)


def test_exemption_flags_near_ties_only():
    lg = np.array([[3.0, 1.0, 1.0 + 1e-9, -2.0], [3.0, 1.0, 0.5, -2.0], [2.0, 2.0, 0.0, -1.0]])
    _, _, ex, _, st = O.route(_cfg(4, 2), lg)
    # row 0: 2nd and 3rd differ by 1e-9 relative; row 2: the two selected tie (order boundary)
    assert ex.tolist() == [True, False, True]
    assert st.exempt_tokens == 2


# ---------------------------------------------------------------- capacity


@pytest.mark.parametrize("case", ["capacity_k1", "capacity_k2", "capacity_drop_when_exhausted", "drop_policy"])
def test_capacity_worked_examples(case):
    g = _gold("routing_worked_examples.json")[case]
    lg = np.array(g["logits"])
    cfg = _cfg(lg.shape[1], g["top_k"], cap_policy=g.get("cap_policy", "overflow_next"),
               capacity=g["capacity"], renormalize=True)
    idx, w, _, st = O.route_capacity(cfg, lg)
    assert idx.tolist() == g["expect_idx"]
    assert st.overflowed == g["expect_overflowed"] and st.dropped == g["expect_dropped"]
    assert (w[idx < 0] == 0).all()


def _fill_event_routing(rankings, k, C):
    """Event-driven reformulation of the greedy: between two fill events every token simply takes
    its first k non-full experts, so commit up to the first token that fills an expert."""
    n, E = rankings.shape
    full = np.zeros(E, bool)
    count = np.zeros(E, np.int64)
    out = -np.ones((n, k), np.int64)
    t0 = 0
    while t0 < n:
        choice = -np.ones((n - t0, k), np.int64)
        for i, t in enumerate(range(t0, n)):
            r = [e for e in rankings[t] if e >= 0 and not full[e]][:k]
            choice[i, : len(r)] = r
        # first token at which some expert reaches C
        run = count.copy()
        stop = n - t0 - 1
        for i in range(n - t0):
            hit = False
            for e in choice[i]:
                if e >= 0:
                    run[e] += 1
                    hit |= run[e] == C
            if hit:
                stop = i
                break
        out[t0 : t0 + stop + 1] = choice[: stop + 1]
        for e in choice[: stop + 1].ravel():
            if e >= 0:
                count[e] += 1
        full |= count >= C
        t0 += stop + 1
    return out


@pytest.mark.parametrize("seed,n,E,k,C", [(8, 16, 4, 2, 5), (9, 300, 8, 2, 60), (10, 400, 16, 3, 50)])
def test_capacity_greedy_matches_fill_event_reformulation(seed, n, E, k, C):
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((n, E)) - 1.2 * np.log(np.arange(E) + 1)  # skewed demand
    cfg = _cfg(E, k, cap_policy="overflow_next", capacity=C)
    idx, w, _, st = O.route_capacity(cfg, lg)
    rankings = np.array([np.lexsort((np.arange(E), -row)) for row in lg])
    np.testing.assert_array_equal(idx, _fill_event_routing(rankings, k, C))
    counts = np.bincount(idx[idx >= 0], minlength=E)
    assert counts.max() <= C
    assert st.overflowed > 0


def test_capacity_at_least_n_times_k_is_no_capacity():
    rng = np.random.default_rng(11)
    lg = rng.standard_normal((500, 16)) - 1.2 * np.log(np.arange(16) + 1)
    i0, w0, _, _, _ = O.route(_cfg(16, 2), lg)
    i1, w1, _, st = O.route_capacity(_cfg(16, 2, cap_policy="overflow_next", capacity=1000), lg)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(w0, w1)
    assert st.overflowed == 0 and st.dropped == 0


def test_capacity_value_formula():
    cfg = _cfg(64, 2, cap_policy="overflow_next", capacity_factor=1.25)
    assert O.capacity_value(cfg, 32768) == 1280  # 1.25 * 32768 * 2 / 64
    assert O.capacity_value(cfg, 1000) == math.ceil(1.25 * 1000 * 2 / 64)


def test_drop_policy_invariants():
    rng = np.random.default_rng(12)
    E, k, C = 16, 2, 40
    lg = rng.standard_normal((600, E)) - 1.2 * np.log(np.arange(E) + 1)
    i0, _, _, _, _ = O.route(_cfg(E, k), lg)
    i1, w1, _, st = O.route_capacity(_cfg(E, k, cap_policy="drop", capacity=C), lg)
    kept = i1 >= 0
    assert (i1[kept] == i0[kept]).all()  # kept slots are the original choices, in place
    counts = np.bincount(i1[kept], minlength=E)
    assert counts.max() <= C and st.dropped == (~kept).sum() > 0
    # a slot is dropped exactly when its expert already had C earlier slots
    seen = np.zeros(E, int)
    for t in range(i0.shape[0]):
        for j in range(k):
            e = i0[t, j]
            assert kept[t, j] == (seen[e] < C)
            seen[e] += kept[t, j]


# ---------------------------------------------------------------- dispatch


def test_dispatch_is_a_stable_argsort():
    rng = np.random.default_rng(13)
    n, k, E = 257, 3, 10
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    idx[5, 1] = -1  # a dropped slot
    counts, offsets, perm, dest = O.dispatch(idx, E)
    flat = idx.ravel()
    keep = np.nonzero(flat >= 0)[0]
    order = keep[np.argsort(flat[keep], kind="stable")]
    np.testing.assert_array_equal(perm, order // k)
    np.testing.assert_array_equal(counts, np.bincount(flat[keep], minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    d = dest.ravel()
    assert d[5 * k + 1] == -1
    np.testing.assert_array_equal(d[order], np.arange(len(order)))  # bijection, inverse of perm


def test_identity_experts_reproduce_input_times_gate_sum():
    w = W.get("deepseek_v3_small")
    inp = W.host_inputs(w, names=["x", "w_r", "bias"])
    cfg = O.Cfg(**w.cfg_fields())
    lg = O.router_logits(inp["x"], inp["w_r"])
    idx, tw, _, _, _ = O.route(cfg, lg, inp["bias"])
    counts, offsets, perm, dest = O.dispatch(idx, w.n_routed)
    x = O.bf16_to_f64(inp["x"])
    y = O.combine(x[perm], dest, tw)  # expert = identity
    np.testing.assert_allclose(y, x * tw.sum(1, keepdims=True), rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- SwiGLU, shared experts, combine


def _torch_swiglu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.from_numpy(O.bf16_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64))
                     for a in (x, wg, wu, wd))
    return (torch.nn.functional.silu(x @ wg.T) * (x @ wu.T) @ wd.T).numpy()


def test_silu_closed_form():
    one = np.ones((1, 1), np.float32)
    out = O.swiglu(np.array([[1.0]]), one, one, one)
    assert out[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)  # silu(1) * 1
    out = O.swiglu(np.array([[-2.0]]), one, one, one)
    assert out[0, 0] == pytest.approx(-2.0 / (1.0 + math.exp(2.0)) * -2.0, rel=1e-15)


def test_swiglu_matches_torch_float64():
    rng = np.random.default_rng(14)
    d, I, m = 48, 80, 9
    x = rng.standard_normal((m, d))
    wg, wu = (rng.standard_normal((I, d)).astype(np.float32) for _ in range(2))
    wd = rng.standard_normal((d, I)).astype(np.float32)
    np.testing.assert_allclose(O.swiglu(x, wg, wu, wd), _torch_swiglu(x, wg, wu, wd), rtol=1e-11, atol=1e-11)


def test_single_expert_layer_is_a_dense_ffn():
    rng = np.random.default_rng(15)
    d, I, n = 32, 48, 20
    x = rng.standard_normal((n, d)).astype(np.float32)
    wr = rng.standard_normal((1, d)).astype(np.float32)
    wg, wu = (rng.standard_normal((1, I, d)).astype(np.float32) for _ in range(2))
    wd = rng.standard_normal((1, d, I)).astype(np.float32)
    cfg = O.Cfg(d_model=d, n_routed=1, top_k=1, moe_intermediate_size=I)
    r = O.layer(cfg, x, wr, wg, wu, wd)
    np.testing.assert_allclose(r["y"], _torch_swiglu(x, wg[0], wu[0], wd[0]), rtol=1e-11, atol=1e-11)


def test_k_equals_E_is_the_dense_softmax_mixture():
    rng = np.random.default_rng(16)
    d, I, n, E = 24, 40, 15, 5
    x = rng.standard_normal((n, d)).astype(np.float32)
    wr = rng.standard_normal((E, d)).astype(np.float32)
    wg, wu = (rng.standard_normal((E, I, d)).astype(np.float32) for _ in range(2))
    wd = rng.standard_normal((E, d, I)).astype(np.float32)
    cfg = O.Cfg(d_model=d, n_routed=E, top_k=E, moe_intermediate_size=I)
    r = O.layer(cfg, x, wr, wg, wu, wd)
    p = scipy.special.softmax(x.astype(np.float64) @ wr.astype(np.float64).T, axis=1)
    ref = sum(p[:, e : e + 1] * _torch_swiglu(x, wg[e], wu[e], wd[e]) for e in range(E))
    np.testing.assert_allclose(r["y"], ref, rtol=1e-10, atol=1e-11)


def test_shared_experts_are_added_unweighted_and_concatenate():
    w = W.get("deepseek_v2_small", n=30)
    inp = W.host_inputs(w)
    cfg = O.Cfg(**w.cfg_fields())
    r = O.layer(cfg, inp["x"], inp["w_r"], inp["w_gate"], inp["w_up"], inp["w_down"],
                ws_gate=inp["ws_gate"], ws_up=inp["ws_up"], ws_down=inp["ws_down"])
    r0 = O.layer(cfg.__class__(**{**cfg.__dict__, "n_shared": 0}), inp["x"], inp["w_r"], inp["w_gate"],
                 inp["w_up"], inp["w_down"])
    I = w.moe_intermediate_size
    sh = sum(_torch_swiglu(inp["x"], inp["ws_gate"][s * I:(s + 1) * I], inp["ws_up"][s * I:(s + 1) * I],
                           inp["ws_down"][:, s * I:(s + 1) * I]) for s in range(w.n_shared))
    np.testing.assert_allclose(r["y"] - r0["y"], sh, rtol=1e-9, atol=1e-10)


def test_layer_composes_route_dispatch_swiglu_combine():
    w = W.get("mixtral_small", n=64)
    inp = W.host_inputs(w)
    cfg = O.Cfg(**w.cfg_fields())
    r = O.layer(cfg, inp["x"], inp["w_r"], inp["w_gate"], inp["w_up"], inp["w_down"])
    lg = O.bf16_to_f64(inp["x"]) @ O.bf16_to_f64(inp["w_r"]).T
    idx = _lexsort_topk(lg, 2)
    np.testing.assert_array_equal(r["topk_idx"], idx)
    sel = np.take_along_axis(lg, idx, 1)
    gw = scipy.special.softmax(sel, axis=1)
    ref = np.zeros((w.n, w.d_model))
    for t in range(w.n):
        for j in range(2):
            e = idx[t, j]
            ref[t] += gw[t, j] * _torch_swiglu(inp["x"][t : t + 1], inp["w_gate"][e], inp["w_up"][e],
                                               inp["w_down"][e])[0]
    np.testing.assert_allclose(r["y"], ref, rtol=1e-9, atol=1e-10)
    np.testing.assert_array_equal(r["counts"], np.bincount(idx.ravel(), minlength=8))


# ---------------------------------------------------------------- V4 routing variants and the bias update


def test_sqrtsoftplus_closed_forms():
    one = lambda l: O.route(_cfg(1, 1, score_fn="sqrtsoftplus"), np.array([[l]]))[1][0, 0]
    assert one(0.0) == pytest.approx(math.sqrt(math.log(2.0)), rel=1e-15)
    assert one(30.0) == pytest.approx(math.sqrt(30.0 + math.log1p(math.exp(-30.0))), rel=1e-15)
    assert one(-30.0) == pytest.approx(math.sqrt(math.log1p(math.exp(-30.0))), rel=1e-12)
    assert one(2.5) == pytest.approx(math.sqrt(math.log(1.0 + math.exp(2.5))), rel=1e-14)


def test_sqrtsoftplus_selection_with_bias_matches_library_sort_and_brute_force():
    rng = np.random.default_rng(21)
    E, k = 12, 3
    lg = rng.standard_normal((300, E)) * 2
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    s = np.sqrt(np.logaddexp(0.0, lg))  # numpy softplus, then sqrt
    c = s + bias.astype(np.float64)
    idx, w, _, _, _ = O.route(_cfg(E, k, score_fn="sqrtsoftplus", renormalize=True, routed_scaling_factor=1.5), lg, bias)
    np.testing.assert_array_equal(idx, _lexsort_topk(c, k))
    sel = np.take_along_axis(s, idx, 1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True) * 1.5, rtol=1e-13)
    # with a group limit the same brute force as for sigmoid applies
    idx2, _, _, _, _ = O.route(_cfg(E, k, score_fn="sqrtsoftplus", n_group=4, topk_group=2), lg, bias)
    for t in range(60):
        assert idx2[t].tolist() == _brute_group_topk(c[t], 4, 2, k), t


def test_hash_routing_uses_the_table_and_scores_only_weight():
    rng = np.random.default_rng(22)
    E, k, vocab, n = 16, 3, 50, 120
    table = np.stack([rng.permutation(E)[:k] for _ in range(vocab)]).astype(np.int32)
    tok = rng.integers(0, vocab, n).astype(np.int32)
    lg = rng.standard_normal((n, E))
    cfg = _cfg(E, k, score_fn="sqrtsoftplus", renormalize=True, routed_scaling_factor=2.0)
    idx, w = O.route_hash(cfg, lg, tok, table)
    np.testing.assert_array_equal(idx, table[tok])
    s = np.sqrt(np.logaddexp(0.0, lg))
    sel = np.take_along_axis(s, idx, 1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True) * 2.0, rtol=1e-13)


def test_bias_update_worked_example():
    g = _gold("routing_worked_examples.json")["bias_update"]
    out = O.bias_update(np.array(g["counts"]), np.array(g["bias"], np.float32), g["gamma"])
    np.testing.assert_allclose(out, g["expect"], rtol=0, atol=1e-12)


# ---- FP8 experts (page "15. DeepSeek: MLA, MoE and MTP", FP8 section) --------------------------

def test_e4m3_published_values():
    """OCP E4M3 facts: largest finite 448, smallest normal 2^-6, smallest subnormal 2^-9, no infinities."""
    t = O.e4m3_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9
    assert t[0x38] == 1.0 and t[0xB8] == -1.0 and t[0x00] == 0.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF]) and np.isnan(t).sum() == 2
    finite = t[:0x7F]
    assert (np.diff(finite) > 0).all()  # codes 0x00..0x7E are increasing


def test_e4m3_codec_matches_torch_float8():
    """Decoding equals torch.float8_e4m3fn for every code; encoding equals torch's round-to-nearest-even
    cast on a sweep that includes every midpoint between neighbouring codes."""
    t = O.e4m3_table()
    codes = torch.arange(256, dtype=torch.uint8)
    tv = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (tv == t) | (np.isnan(tv) & np.isnan(t))
    assert same.all()
    pos = t[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(1)
    sweep = np.concatenate([pos, mids, rng.uniform(0, 448, 2000), rng.uniform(0, 2 ** -6, 500)])
    sweep = np.concatenate([sweep, -sweep]).astype(np.float32)  # all exact in binary32
    ref = torch.from_numpy(sweep).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode(float(v)) for v in sweep], np.uint8)
    np.testing.assert_array_equal(got, ref)
    assert O.e4m3_encode(1e6) == 0x7E and O.e4m3_encode(-449.0) == 0xFE  # saturation (reading)


def test_ue8m0_exponent_is_the_smallest_power_of_two_that_fits():
    rng = np.random.default_rng(2)
    vals = list(rng.lognormal(0, 6, 3000)) + [448.0 * 2.0 ** k for k in range(-20, 20)]
    vals += [np.nextafter(448.0 * 2.0 ** k, np.inf) for k in range(-20, 20)]
    for a in vals:
        e = O.ue8m0_exponent(a)
        assert a <= 448.0 * 2.0 ** e and a > 448.0 * 2.0 ** (e - 1), (a, e)
    assert O.ue8m0_exponent(0.0) == 0


def test_quantize_rows_tiles_scales_and_codes():
    rng = np.random.default_rng(3)
    a = rng.normal(0, 1, (7, 384)) * rng.lognormal(0, 3, (7, 1))
    a[2, 128:256] = 0.0  # an all-zero tile
    codes, sb = O.quantize_rows(a)
    assert codes.shape == a.shape and sb.shape == (7, 3)
    for r in range(7):
        for t in range(3):
            tile = a[r, 128 * t:128 * (t + 1)]
            e = int(sb[r, t]) - 127
            amax = np.abs(tile).max()
            assert (amax == 0 and e == 0) or (amax <= 448 * 2.0 ** e < 2 * amax)
            scaled = torch.from_numpy(tile * 2.0 ** -e)  # exact power-of-two scaling
            ref = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            np.testing.assert_array_equal(codes[r, 128 * t:128 * (t + 1)], ref)


def test_dequant_blocks_on_constructed_weights():
    """All codes 1.0 and a distinct scale per 128 x 128 block: each block must come out as its own power of two."""
    N, K = 300, 384
    codes = np.full((N, K), 0x38, np.uint8)
    sb = (120 + np.arange(3 * 3).reshape(3, 3)).astype(np.uint8)
    w = O.dequant_blocks(codes, sb)
    for bi in range(3):
        for bj in range(3):
            blk = w[128 * bi:128 * (bi + 1), 128 * bj:128 * (bj + 1)]
            assert (blk == 2.0 ** (int(sb[bi, bj]) - 127)).all()


def test_fp8_layer_equals_bf16_layer_when_quantisation_is_lossless():
    """Ternary activations and weights (exact in E4M3 with unit-like scales) whose SwiGLU outputs stay
    exact: with W_gate = W_up = 0 the hidden values are 0 (exact), so the FP8 layer must equal the bf16
    layer on the dequantised weights; with ternary x the first quantisation is exact as well."""
    w = W.get("tie_softmax", d_model=128, moe_intermediate_size=128, n=64)
    host = W.host_inputs(w)
    E, I, d = w.n_routed, w.moe_intermediate_size, w.d_model
    rng = np.random.default_rng(4)
    zero = (np.zeros((E, I, d), np.uint8), np.full((E, 1, 1), 127, np.uint8))
    down = (rng.choice(np.array([0x38, 0xB8, 0x00], np.uint8), (E, d, I)), np.full((E, 1, 1), 120, np.uint8))
    r8 = O.layer_fp8(O.Cfg(**w.cfg_fields()), host["x"], host["w_r"], None, dict(gate=zero, up=zero, down=down))
    assert np.abs(r8["y"]).max() == 0.0
    # Non-zero gate/up: compare the experts' hidden layer directly against torch's float8 cast.
    x64 = O.bf16_to_f64(host["x"])
    xq, xs = O.quantize_rows(x64)
    np.testing.assert_array_equal(O.dequant_rows(xq, xs), x64)  # ternary rows quantise exactly


def test_fp8_layer_close_to_unquantised_layer():
    """FP8 quantisation of x and h changes the layer by a few per cent at most (E4M3 keeps 4 significant
    bits: relative rounding error <= 2^-4 per element), not by orders of magnitude."""
    w = W.get("fp8_ragged_small")
    host = W.host_inputs(w)
    w8 = {k: (host["w_%s_q" % k], host["w_%s_s" % k]) for k in ("gate", "up", "down")}
    ws8 = {k: (host["ws_%s_q" % k], host["ws_%s_s" % k]) for k in ("gate", "up", "down")}
    r8 = O.layer_fp8(O.Cfg(**w.cfg_fields()), host["x"], host["w_r"], None, w8, ws8)
    deq = lambda q, s: np.stack([O.dequant_blocks(q[e], s[e]) for e in range(q.shape[0])]).astype(np.float32)
    ref = O.layer(O.Cfg(**w.cfg_fields()), O.bf16_to_f64(host["x"]).astype(np.float32),
                  O.bf16_to_f64(host["w_r"]).astype(np.float32), deq(*w8["gate"]), deq(*w8["up"]),
                  deq(*w8["down"]), None, *(O.dequant_blocks(*ws8[k]).astype(np.float32) for k in ("gate", "up", "down")))
    np.testing.assert_array_equal(r8["topk_idx"], ref["topk_idx"])
    err = np.sqrt(((r8["y"] - ref["y"]) ** 2).mean() / (ref["y"] ** 2).mean())
    assert 1e-4 < err < 0.05, err


def test_round_to_bf16_matches_torch_on_binary32_values():
    """On values that binary32 holds exactly, one rounding to bf16 is torch's binary32 -> bf16 cast."""
    rng = np.random.default_rng(5)
    a = np.concatenate([rng.normal(0, 1, 5000) * rng.lognormal(0, 4, 5000), [0.0, -0.0, 1.0, 3.0 / 7.0,
                        2.0 ** -130, -3 * 2.0 ** -133, 2.0 ** 127 * 1.5]])
    a = a.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to_bf16(a), ref)


def test_round_to_bf16_rounds_once_from_binary64():
    """Ties go to the even neighbour; a value a hair above a tie (2^-30 relative, below binary32's
    resolution) rounds up, which a rounding through binary32 would get wrong; the grid at
    [64, 128) is 1/2."""
    v = np.array([68.25, 68.75, 68.25 + 2.0 ** -24, 68.25 - 2.0 ** -24, -68.25 - 2.0 ** -24, 1.0 + 2.0 ** -8,
                  1.0 + 3 * 2.0 ** -8, 2.0 ** -126 * (1 + 2.0 ** -8)])
    want = np.array([68.0, 69.0, 68.5, 68.0, -68.5, 1.0, 1.0 + 2.0 ** -6, 2.0 ** -126])
    np.testing.assert_array_equal(O.round_to_bf16(v), want)
    via32 = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert via32[2] == 68.0  # the double rounding that the one-step rounding avoids


def test_swiglu_fp8_hidden_step_on_constructed_boundaries():
    """The h step of the FP8 expert, exactly: x has four unit entries (quantised exactly), gate rows
    give g = 64 (silu(64) = 64 in binary64), up rows give u as a sum of four E4M3 values in three
    k-blocks (the last with scale 2^-21), so h = 64 u is known exactly; W_down is the identity on the
    first 128 outputs, so the layer returns the dequantised E4M3 codes of h. Expected values by hand:
    448 sets the tile's scale to 2^0; 68.25 + 2^-24 -> bf16 68.5 -> E4M3 72; 68.25 -> bf16 68 (tie to
    even) -> E4M3 64 (tie to even; the binary64 value would give 72); 69 -> 72; 67.75 -> bf16 68 ->
    E4M3 64; 76 -> E4M3 80 (tie to even)."""
    d, I = 384, 128
    enc = np.vectorize(O.e4m3_encode, otypes=[np.uint8])
    x = np.zeros((1, d))
    x[0, [0, 1, 128, 256]] = 1.0
    wg = np.zeros((I, d))
    wg[:, 0] = 64.0
    u_terms = {0: (7.0, 0, 0, 0),
               1: (1.0, 2.0 ** -4, 2.0 ** -8, 2.0 ** -30),
               2: (1.0, 2.0 ** -4, 2.0 ** -8, 0),
               3: (1.0, 2.0 ** -4, 2.0 ** -6, 0),
               4: (1.0, 2.0 ** -4, -(2.0 ** -8), 0),
               5: (1.0, 0.1875, 0, 0)}
    wu = np.zeros((I, d))
    for i, (a, b, c, e) in u_terms.items():
        wu[i, 0], wu[i, 1], wu[i, 128], wu[i, 256] = a, b, c, e
    sc_u = np.array([[127, 127, 127 - 21]], np.uint8)
    codes_u = np.zeros((I, d), np.uint8)
    for blk in range(3):
        cols = slice(128 * blk, 128 * (blk + 1))
        codes_u[:, cols] = enc(wu[:, cols] * 2.0 ** -(int(sc_u[0, blk]) - 127))
    np.testing.assert_array_equal(O.dequant_blocks(codes_u, sc_u), wu)  # the constructed u terms are exact
    wd = np.zeros((d, I))
    wd[np.arange(I), np.arange(I)] = 1.0
    ones = lambda r, c: np.full((r, c), 127, np.uint8)
    out = O.swiglu_fp8(x, (enc(wg), ones(1, 3)), (codes_u, sc_u), (enc(wd), ones(3, 1)))
    want = np.zeros((1, d))
    want[0, :6] = [448.0, 72.0, 64.0, 72.0, 64.0, 80.0]
    np.testing.assert_array_equal(out, want)


# ---------------------------------------------------------------- expert parallelism: receive layout


@pytest.mark.parametrize("world,E,k", [(1, 8, 2), (2, 8, 2), (4, 16, 3), (8, 64, 6)])
def test_ep_recv_layout_is_the_global_stable_permutation_split_by_owner(world, E, k):
    """Pinned to the oracle's C counting sort of the concatenated batch (a separate formulation):
    the owners' rows, concatenated in owner order, are its permutation, and each owner's expert
    ranges are its offsets shifted to start at zero."""
    rng = np.random.default_rng(world * 100 + E)
    ns = [int(v) for v in rng.integers(0, 40, world)]
    ns[0] = 0 if world > 1 else ns[0]  # a rank without tokens
    idx = [np.array([rng.choice(E, k, replace=False) for _ in range(n)], np.int32).reshape(n, k) for n in ns]
    if world > 1:  # a dropped slot (-1) is never received
        idx[-1][:1, -1] = -1
    lay = O.ep_recv_layout(idx, E, world)
    _, off, perm, _ = O.dispatch(np.concatenate(idx), E)
    first = np.cumsum([0] + ns)
    glob = np.concatenate([first[rows[:, 0]] + rows[:, 1] for rows, _ in lay])
    np.testing.assert_array_equal(glob, perm)
    Eq = E // world
    for q, (_, offs) in enumerate(lay):
        np.testing.assert_array_equal(offs, off[q * Eq:(q + 1) * Eq + 1] - off[q * Eq])
