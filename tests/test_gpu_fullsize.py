"""Parity at the full workload sizes, in the configuration the benchmark runs.

The GPU runs the whole batch; the oracle recomputes sampled tokens one by one
(routing, every selected expert's SwiGLU with that expert's weights
regenerated on the host, shared experts, combine). Under a capacity limit the
oracle routes the whole batch, since the rule is sequential in token order.
Whole-batch properties are checked at every size: counts equal the histogram
of the returned indices, every token holds k distinct experts, and the
permutation is a bijection.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from synth import workloads as W
from tests import moe_harness as H

pytestmark = pytest.mark.gpu

FULL = ["tiny_f32", "mixtral_8x7b", "deepseek_v2", "deepseek_v3_prefill", "deepseek_v3_decode", "skewed_capacity"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _oracle_token(w, host_wr, bias, x_row, idx_row, w_row):
    """y for one token from the oracle's routing of that token."""
    d, I = w.d_model, w.moe_intermediate_size
    x64 = O.bf16_to_f64(x_row)[None, :]
    y = np.zeros(d)
    for e, g in zip(idx_row, w_row):
        if e < 0:
            continue
        wg = W.host_rows(w, "w_gate", [e])[0]
        wu = W.host_rows(w, "w_up", [e])[0]
        wd = W.host_rows(w, "w_down", [e])[0]
        y += g * O.swiglu(x64, wg, wu, wd)[0]
    if w.n_shared:
        sh = W.host_inputs(w, names=["ws_gate", "ws_up", "ws_down"])
        y += O.swiglu(x64, sh["ws_gate"], sh["ws_up"], sh["ws_down"])[0]
    return y


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
    host_wr = W.host_inputs(w, names=["w_r"] + (["bias"] if w.bias_range else []))
    bias = host_wr.get("bias")
    ocfg = H.oracle_cfg(w)
    rng = np.random.default_rng(0)
    samples = sorted({0, w.n - 1, *rng.integers(0, w.n, 4).tolist()})
    if w.cap_policy != "none":
        x_all = W.host_inputs(w, names=["x"])["x"]
        oi, ow, ex, st = O.route_capacity(ocfg, O.router_logits(x_all, host_wr["w_r"]), bias)
        stop = int(np.argmax(ex)) if ex.any() else w.n
        np.testing.assert_array_equal(gi[:stop], oi[:stop])
        if stop == w.n:
            assert diag["overflowed"] == st.overflowed and diag["dropped"] == st.dropped
        samples = [t for t in samples if t < stop]
        xs = x_all[samples]
        oi_s, ow_s = oi[samples], ow[samples]
        ex_s = np.zeros(len(samples), bool)
    else:
        xs = W.host_rows(w, "x", samples)
        oi_s, ow_s, ex_s, _, _ = O.route(ocfg, O.router_logits(xs, host_wr["w_r"]), bias)
        keep = ~ex_s
        np.testing.assert_array_equal(gi[samples][keep], oi_s[keep])
        np.testing.assert_allclose(gw[samples][keep], ow_s[keep], rtol=2e-4, atol=1e-6)
    y = H.as_f64(got["y"][samples])
    for i, t in enumerate(samples):
        if ex_s[i]:
            continue
        ref = _oracle_token(w, host_wr["w_r"], bias, xs[i], oi_s[i], ow_s[i])
        assert H.rel_err(y[i], ref) <= H.TOL[w.dtype], (name, t)
