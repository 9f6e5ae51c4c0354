"""Shared helpers of the GPU parity tests: device inputs, calls through the C ABI,
the oracle side on the host, and the comparison metrics."""
from __future__ import annotations

import numpy as np
import torch

import top_routing_expert_router_b200 as moe
from oracle import oracle as O
from synth import workloads as W

TOL = {"bf16": 2e-2, "f32": 1e-4}


def cfg_for(w: W.Workload):
    return moe.make_config(dtype=w.dtype, **{k: v for k, v in w.cfg_fields().items()})


def oracle_cfg(w: W.Workload):
    return O.Cfg(**w.cfg_fields())


def weights_for(inp: dict):
    return moe.make_weights(inp["w_r"], inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                            inp.get("ws_up"), inp.get("ws_down"), inp.get("bias"))


def workspace(cfg, n, device="cuda"):
    nbytes = moe.moe_workspace_size(cfg, n)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def to_np(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host array in the oracle's encoding (float32 or raw bf16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def as_f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return O.bf16_to_f64(t)


def rel_err(y: np.ndarray, r: np.ndarray) -> float:
    """max over elements of |y - r| / max(|r|, rms of r over the same token's row).

    "Max relative error" is undefined where r ~ 0; the floor is the token's own
    output scale (the row rms), so that tokens with small gates (e.g. capacity
    overflow onto low-probability experts) are measured against their own size.
    """
    if not r.size:
        return 0.0
    r2 = r.reshape(-1, r.shape[-1]) if r.ndim > 1 else r.reshape(1, -1)
    y2 = y.reshape(r2.shape)
    rms = np.sqrt(np.mean(r2 * r2, axis=1, keepdims=True))
    rms[rms == 0] = 1.0
    return float(np.max(np.abs(y2 - r2) / np.maximum(np.abs(r2), rms)))


def run_layer(w: W.Workload, inp: dict, n=None, diag=True):
    n = w.n if n is None else n
    cfg = cfg_for(w)
    ws = workspace(cfg, n)
    dev = inp["x"].device
    y = torch.empty((n, w.d_model), dtype=inp["x"].dtype, device=dev)
    idx = torch.empty((n, w.top_k), dtype=torch.int32, device=dev)
    tw = torch.empty((n, w.top_k), dtype=torch.float32, device=dev)
    counts = torch.empty(w.n_routed, dtype=torch.int32, device=dev)
    dg = torch.zeros(8, dtype=torch.int32, device=dev) if diag else None
    weights = weights_for(inp)
    moe.moe_layer_forward(cfg, n, inp["x"], weights, y, ws, idx, tw, counts, dg)
    st = moe.moe_sync_status(ws)
    assert st == moe.MOE_OK, moe.moe_status_string(st)
    return dict(y=y, topk_idx=idx, topk_w=tw, counts=counts, diag=dg)


def diag_dict(dg: torch.Tensor) -> dict:
    v = dg.cpu().tolist()
    return dict(zip(moe.DIAG_FIELDS, v))


def first_mismatch(a: np.ndarray, b: np.ndarray) -> int:
    bad = np.nonzero((a != b).reshape(a.shape[0], -1).any(1))[0]
    return int(bad[0]) if bad.size else -1
