"""Named workloads (layer shapes and routing settings) and the seeded input recipe.

Full-size workloads are shaped like the models on the pages (Mixtral-8x7B,
DeepSeek-V2, DeepSeek-V3 prefill/decode) plus a tiny fp32 case and a skewed,
capacity-limited case. The ``*_small`` workloads keep each one's routing
structure at sizes the fp64 oracle finishes in seconds while still spanning
several GEMM tiles with ragged tails. ``tie_*`` workloads use ternary inputs so
that router logits are small integers with exact ties.

Input recipe (seed 0 unless stated): x ~ N(0,1); W_r ~ N(0, 1/d); W_gate,
W_up ~ N(0, 1/d); W_down ~ N(0, 1/I); shared experts likewise (W_down fan-in
I per shared expert); selection bias ~ U(-0.1, 0.1) where the router uses it.
N(0, s^2) is the Irwin-Hall(12) construction of ``synth.h``. The skewed
workload adds the per-expert offset -s*ln(e+1) (s = 1.2) to every router
logit through a constant feature: x[:, d-1] = 1 and W_r[e, d-1] = offset_e.
This module holds no arithmetic of the MoE layer.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    n: int
    d_model: int
    n_routed: int
    top_k: int
    moe_intermediate_size: int
    n_shared: int = 0
    n_group: int = 1
    topk_group: int = 1
    score_fn: str = "softmax"
    renormalize: bool = False
    routed_scaling_factor: float = 1.0
    cap_policy: str = "none"
    capacity_factor: float = 0.0
    capacity: int = 0
    dtype: str = "bf16"
    bias_range: tuple | None = None
    zipf_s: float = 0.0
    ternary: bool = False
    router_scale: float = 1.0  # multiplies the router weights' standard deviation (logit stress cases)
    description: str = ""

    @property
    def I_s(self) -> int:
        return self.n_shared * self.moe_intermediate_size

    def cfg_fields(self) -> dict:
        """The layer configuration in the pages' field names."""
        return dict(
            d_model=self.d_model, n_routed=self.n_routed, top_k=self.top_k,
            moe_intermediate_size=self.moe_intermediate_size, n_shared=self.n_shared,
            n_group=self.n_group, topk_group=self.topk_group, score_fn=self.score_fn,
            renormalize=self.renormalize, routed_scaling_factor=self.routed_scaling_factor,
            cap_policy=self.cap_policy, capacity_factor=self.capacity_factor, capacity=self.capacity,
        )

    def tensor_specs(self) -> dict:
        """name -> (shape, stream, kind, a, b, dtype)."""
        d, E, I, Is = self.d_model, self.n_routed, self.moe_intermediate_size, self.I_s
        dt = self.dtype
        kind_x = synth.TERNARY if self.ternary else synth.NORMAL
        specs = {
            "x": ((self.n, d), synth.STREAM["x"], kind_x, 1.0, 0.0, dt),
            "w_r": ((E, d), synth.STREAM["w_r"], kind_x, self.router_scale / math.sqrt(d), 0.0, dt),
            "w_gate": ((E, I, d), synth.STREAM["w_gate"], synth.NORMAL, 1.0 / math.sqrt(d), 0.0, dt),
            "w_up": ((E, I, d), synth.STREAM["w_up"], synth.NORMAL, 1.0 / math.sqrt(d), 0.0, dt),
            "w_down": ((E, d, I), synth.STREAM["w_down"], synth.NORMAL, 1.0 / math.sqrt(I), 0.0, dt),
        }
        if self.bias_range is not None:
            lo, hi = self.bias_range
            specs["bias"] = ((E,), synth.STREAM["bias"], synth.UNIFORM, lo, hi, "f32")
        if self.n_shared > 0:
            specs["ws_gate"] = ((Is, d), synth.STREAM["ws_gate"], synth.NORMAL, 1.0 / math.sqrt(d), 0.0, dt)
            specs["ws_up"] = ((Is, d), synth.STREAM["ws_up"], synth.NORMAL, 1.0 / math.sqrt(d), 0.0, dt)
            specs["ws_down"] = ((d, Is), synth.STREAM["ws_down"], synth.NORMAL, 1.0 / math.sqrt(I), 0.0, dt)
        if dt == "fp8":
            # FP8 experts: activations and router stay bf16; every expert matrix is E4M3 codes plus one
            # UE8M0 scale byte per 128 x 128 block, drawn directly as bytes (no conversion arithmetic).
            for nm in ("x", "w_r"):
                specs[nm] = specs[nm][:5] + ("bf16",)
            for nm in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
                if nm not in specs:
                    continue
                shape = specs.pop(nm)[0]
                fan_in = shape[-1]
                lo, hi = _fp8_scale_bytes(fan_in)
                sshape = shape[:-2] + (-(-shape[-2] // 128), shape[-1] // 128)
                specs[nm + "_q"] = (shape, synth.STREAM[nm + "_q"], synth.SIGNED_CODE, FP8_CODE_LO, FP8_CODE_HI, "u8")
                specs[nm + "_s"] = (sshape, synth.STREAM[nm + "_s"], synth.BYTE, lo, hi, "u8")
        return specs


# FP8 weight codes: sign plus a magnitude code uniform on [0x28, 0x47], i.e. E4M3 values of magnitude
# 0.25 .. 3.75 (exponent fields 5..8, all mantissas); their root mean square is about 1.69.
FP8_CODE_LO, FP8_CODE_HI, FP8_CODE_RMS = 0x28, 0x47, 1.69


def _fp8_scale_bytes(fan_in: int) -> tuple:
    """UE8M0 scale bytes (e + 127) of the two powers of two around 1 / (1.69 sqrt(fan_in)), so that the
    weights' root mean square is close to 1/sqrt(fan_in) like the bf16 recipe."""
    e = math.floor(math.log2(1.0 / (FP8_CODE_RMS * math.sqrt(fan_in))))
    return e + 127, e + 128


def _wl(name, **kw) -> Workload:
    return Workload(name=name, **kw)


_V3 = dict(d_model=7168, n_routed=256, n_shared=1, top_k=8, moe_intermediate_size=2048,
           score_fn="sigmoid", n_group=8, topk_group=4, renormalize=True, routed_scaling_factor=2.5,
           bias_range=(-0.1, 0.1))

WORKLOADS = {w.name: w for w in [
    _wl("tiny_f32", n=64, d_model=128, n_routed=8, top_k=2, moe_intermediate_size=256, dtype="f32",
        description="tiny softmax top-2, fp32"),
    _wl("mixtral_8x7b", n=4096, d_model=4096, n_routed=8, top_k=2, moe_intermediate_size=14336,
        renormalize=True, description="Mixtral-8x7B-shaped, softmax top-2, renormalised gates"),
    _wl("deepseek_v2", n=8192, d_model=5120, n_routed=160, n_shared=2, top_k=6,
        moe_intermediate_size=1536, description="DeepSeek-V2-shaped, softmax top-6, 2 shared"),
    _wl("deepseek_v3_prefill", n=16384, description="DeepSeek-V3-shaped prefill", **_V3),
    _wl("deepseek_v3_decode", n=64, description="DeepSeek-V3-shaped decode", **_V3),
    _wl("skewed_capacity", n=32768, d_model=4096, n_routed=64, top_k=2, moe_intermediate_size=2048,
        cap_policy="overflow_next", capacity_factor=1.25, zipf_s=1.2,
        description="skewed softmax top-2, capacity 1.25*n*k/E, overflow to next-best"),
    # profiling case: Mixtral shapes with 4 experts (1.4 GB of weights, still far larger than L2)
    _wl("mixtral_4e", n=2048, d_model=4096, n_routed=4, top_k=2, moe_intermediate_size=14336,
        renormalize=True, description="Mixtral-shaped layer with 4 experts (profiling size)"),
    # parity-size variants
    _wl("mixtral_small", n=700, d_model=256, n_routed=8, top_k=2, moe_intermediate_size=384,
        renormalize=True),
    _wl("deepseek_v2_small", n=500, d_model=320, n_routed=160, n_shared=2, top_k=6,
        moe_intermediate_size=192),
    _wl("deepseek_v3_small", n=333, **{**_V3, "d_model": 256, "moe_intermediate_size": 128}),
    _wl("deepseek_v3_decode_small", n=40, **{**_V3, "d_model": 512, "moe_intermediate_size": 256}),
    _wl("skewed_small", n=2000, d_model=256, n_routed=64, top_k=2, moe_intermediate_size=128,
        cap_policy="overflow_next", capacity_factor=1.25, zipf_s=1.2),
    _wl("drop_small", n=1000, d_model=128, n_routed=16, top_k=2, moe_intermediate_size=64,
        cap_policy="drop", capacity_factor=1.0, zipf_s=1.2),
    _wl("ragged_small", n=77, d_model=200, n_routed=5, top_k=2, moe_intermediate_size=72, renormalize=True,
        n_shared=1),
    _wl("deepseek_v4_small", n=300, d_model=256, n_routed=64, n_shared=1, top_k=6, moe_intermediate_size=128,
        score_fn="sqrtsoftplus", renormalize=True, bias_range=(-0.1, 0.1),
        description="DeepSeek-V4-style routing: sqrtsoftplus scores + bias, no group limit"),
    # FP8 experts (DeepSeek-V3 checkpoint format: E4M3 with UE8M0 128 x 128 block scales)
    _wl("deepseek_v3_prefill_fp8", n=16384, dtype="fp8", description="DeepSeek-V3-shaped prefill, FP8 experts", **_V3),
    _wl("deepseek_v3_decode_fp8", n=64, dtype="fp8", description="DeepSeek-V3-shaped decode, FP8 experts", **_V3),
    _wl("deepseek_v3_small_fp8", n=333, dtype="fp8", **{**_V3, "d_model": 256, "moe_intermediate_size": 128}),
    _wl("fp8_ragged_small", n=300, d_model=384, n_routed=12, top_k=3, moe_intermediate_size=256, n_shared=1,
        dtype="fp8", renormalize=True),
    _wl("deepseek_v3_decode_small_fp8", n=40, dtype="fp8", **{**_V3, "d_model": 512, "moe_intermediate_size": 256}),
    # profiling cases of the HBM-bound kernels at DeepSeek-V3 shapes, a few GB on the device:
    # routing and permutation of 8192 tokens (experts shrunk to I = 128: the router and the
    # dispatch do not depend on I), and decode with 32 bf16 experts (2.8 GB of weights)
    _wl("deepseek_v3_route_8k", n=8192, description="DeepSeek-V3 routing and dispatch, small experts (profiling size)",
        **{**_V3, "moe_intermediate_size": 128}),
    # the full layer's router input (x: 235 MB, more than L2) with small experts: router profiling
    _wl("deepseek_v3_route_16k", n=16384, description="DeepSeek-V3 routing and dispatch at 16384 tokens, small experts "
        "(router profiling size)", **{**_V3, "moe_intermediate_size": 128}),
    _wl("deepseek_v3_decode_32e", n=64, description="DeepSeek-V3-shaped decode with 32 experts (profiling size)",
        **{**_V3, "n_routed": 32, "n_group": 8, "topk_group": 4}),
    # profiling case: DeepSeek-V3 prefill shapes with 32 bf16 experts (2.8 GB of weights, 512 rows per
    # expert on average like the full layer, so DRAM traffic per routed slot matches it)
    _wl("deepseek_v3_prefill_32e", n=2048, **{**_V3, "n_routed": 32, "n_group": 8, "topk_group": 4},
        description="DeepSeek-V3-shaped prefill with 32 bf16 experts (profiling size)"),
    # profiling case: DeepSeek-V3 prefill shapes with 32 FP8 experts (1.4 GB of weights, 512 rows
    # per expert: the SM-pair FP8 tiles)
    _wl("deepseek_v3_prefill_fp8_32e", n=2048, dtype="fp8",
        **{**_V3, "n_routed": 32, "n_group": 8, "topk_group": 4},
        description="DeepSeek-V3-shaped prefill with 32 FP8 experts (profiling size)"),
    # profiling case: DeepSeek-V3 decode shapes with 32 FP8 experts (1.4 GB of weights)
    _wl("deepseek_v3_decode_fp8_32e", n=64, dtype="fp8",
        **{**_V3, "n_routed": 32, "n_group": 8, "topk_group": 4},
        description="DeepSeek-V3-shaped decode with 32 FP8 experts (profiling size)"),
    _wl("fp8_skewed_small", n=200, d_model=256, n_routed=16, top_k=1, moe_intermediate_size=128, zipf_s=1.2,
        dtype="fp8"),
    # router stress cases at d = 7168 (routing only): logits 8x (sigmoid, V3 groups) and 4x (softmax,
    # no groups) the recipe's scale, so the binary32 logit errors are as large as they get here
    _wl("deepseek_v3_route_x8", n=16384, router_scale=8.0,
        description="DeepSeek-V3 routing with router weights 8x the recipe's scale", **_V3),
    _wl("softmax_7168_route_x4", n=16384, d_model=7168, n_routed=256, top_k=8, moe_intermediate_size=128,
        router_scale=4.0, description="softmax top-8 of 256 experts at d = 7168, router weights 4x the recipe's scale"),
    _wl("tie_softmax", n=256, d_model=64, n_routed=16, top_k=4, moe_intermediate_size=64,
        ternary=True, renormalize=True),
    _wl("tie_sigmoid", n=256, d_model=64, n_routed=32, top_k=4, moe_intermediate_size=64,
        score_fn="sigmoid", n_group=4, topk_group=2, renormalize=True, routed_scaling_factor=2.5,
        ternary=True),
]}


def get(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def zipf_offsets(w: Workload) -> np.ndarray:
    """Per-expert router-logit offsets -s*ln(e+1) (float64)."""
    return np.array([-w.zipf_s * math.log(e + 1) for e in range(w.n_routed)], np.float64)


def _to_dtype(v64: np.ndarray, dt: str) -> np.ndarray:
    f = v64.astype(np.float32)
    if dt == "f32":
        return f
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def host_tensor(w: Workload, name: str, seed: int = 0, start: int = 0, count: int | None = None):
    """Flat elements [start, start + count) of one input tensor on the host (patched as the recipe says)."""
    shape, stream, kind, a, b, dt = w.tensor_specs()[name]
    total = int(np.prod(shape))
    count = total - start if count is None else count
    out = synth.host((count,), dt, seed, stream, kind, a, b, start)
    if w.zipf_s and name in ("x", "w_r"):
        d = w.d_model
        first_row = start // d
        last_row = (start + count - 1) // d
        for r in range(first_row, last_row + 1):
            j = r * d + d - 1 - start
            if 0 <= j < count:
                if name == "x":
                    out[j] = _to_dtype(np.array([1.0]), dt)[0]
                else:
                    out[j] = _to_dtype(zipf_offsets(w)[r : r + 1], dt)[0]
    return out


def host_inputs(w: Workload, seed: int = 0, names=None) -> dict:
    """Whole input tensors on the host, shaped."""
    specs = w.tensor_specs()
    names = names or list(specs)
    return {nm: host_tensor(w, nm, seed).reshape(specs[nm][0]) for nm in names}


def host_rows(w: Workload, name: str, rows, seed: int = 0) -> np.ndarray:
    """Selected leading-index slices (e.g. token rows of x, experts of W_gate), stacked."""
    shape = w.tensor_specs()[name][0]
    per = int(np.prod(shape[1:]))
    return np.stack([host_tensor(w, name, seed, int(r) * per, per).reshape(shape[1:]) for r in rows])


def device_inputs(w: Workload, seed: int = 0, device="cuda", names=None) -> dict:
    """Whole input tensors created directly in device memory."""
    import torch

    specs = w.tensor_specs()
    names = names or list(specs)
    out = {}
    for nm in names:
        shape, stream, kind, a, b, dt = specs[nm]
        t = torch.empty(shape, dtype={"f32": torch.float32, "bf16": torch.bfloat16, "u8": torch.uint8}[dt],
                        device=device)
        synth.device(t, seed, stream, kind, a, b)
        if w.zipf_s and nm in ("x", "w_r"):
            if nm == "x":
                t[:, -1] = 1.0
            else:
                col = _to_dtype(zipf_offsets(w), dt)
                if dt == "f32":
                    t[:, -1] = torch.from_numpy(col).to(device)
                else:
                    t.view(torch.int16)[:, -1] = torch.from_numpy(col.view(np.int16)).to(device)
        out[nm] = t
    return out
