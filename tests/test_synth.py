"""The seeded input generator: determinism, slicing, moments and bf16 rounding."""
import numpy as np
import torch

from synth import synth, workloads as W


def test_deterministic_and_seeded():
    a = synth.host((1000,), "f32", 0, 1, synth.NORMAL, 1.0)
    b = synth.host((1000,), "f32", 0, 1, synth.NORMAL, 1.0)
    c = synth.host((1000,), "f32", 1, 1, synth.NORMAL, 1.0)
    d = synth.host((1000,), "f32", 0, 2, synth.NORMAL, 1.0)
    assert (a == b).all() and not (a == c).all() and not (a == d).all()


def test_any_slice_equals_the_slice_of_the_whole():
    whole = synth.host((5000,), "bf16", 3, 4, synth.NORMAL, 0.5)
    part = synth.host((777,), "bf16", 3, 4, synth.NORMAL, 0.5, start=1234)
    assert (whole[1234:1234 + 777] == part).all()


def test_irwin_hall_moments_and_support():
    v = synth.host((400000,), "f32", 0, 1, synth.NORMAL, 1.0).astype(np.float64)
    assert abs(v.mean()) < 0.01 and abs(v.var() - 1.0) < 0.01
    assert v.min() >= -6.0 and v.max() <= 6.0
    # kurtosis of Irwin-Hall(12) is 3 - 1.2/12 = 2.9
    k = ((v - v.mean()) ** 4).mean() / v.var() ** 2
    assert abs(k - 2.9) < 0.03


def test_uniform_and_ternary():
    u = synth.host((100000,), "f32", 0, 3, synth.UNIFORM, -0.1, 0.1).astype(np.float64)
    assert u.min() >= -0.1 and u.max() < 0.1 and abs(u.mean()) < 2e-3
    t = synth.host((30000,), "f32", 0, 3, synth.TERNARY, 0.0)
    assert set(np.unique(t).tolist()) == {-1.0, 0.0, 1.0}


def test_bf16_is_round_to_nearest_even_of_the_f32_value():
    f = synth.host((100000,), "f32", 5, 6, synth.NORMAL, 0.01)
    b = synth.host((100000,), "bf16", 5, 6, synth.NORMAL, 0.01)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (b == ref).all()


def test_skew_patch_on_host_rows():
    w = W.get("skewed_small")
    x = W.host_rows(w, "x", [0, 7, 1999])
    wr = W.host_inputs(w, names=["w_r"])["w_r"]
    assert (x[:, -1] == 0x3F80).all()  # bf16 bits of 1.0
    off = (wr[:, -1].astype(np.uint32) << 16).view(np.float32)
    np.testing.assert_allclose(off, -1.2 * np.log(np.arange(64) + 1), rtol=4e-3)
    # whole-tensor and row generation agree
    full = W.host_inputs(w, names=["x"])["x"]
    assert (full[[0, 7, 1999]] == x).all()
