"""Python binding of the B200 sparse-MoE FFN layer library (``libmoe_b200.so``).

Argument marshalling only: every function forwards device pointers, sizes and
the current CUDA stream to the C entry point of the same name declared in
``include/moe.h``. All computation runs in the library's CUDA kernels. Importing
this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python top_routing_expert_router_b200/build.py` "
                      "(or __graft_entry__.build()); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, \
    MOE_ERR_INTERNAL = range(7)
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID, MOE_SCORE_SQRTSOFTPLUS = 0, 1, 2
MOE_CAP_NONE, MOE_CAP_OVERFLOW_NEXT, MOE_CAP_DROP = 0, 1, 2
MOE_F32, MOE_BF16, MOE_FP8 = 0, 1, 2

# Every symbol declared in include/moe.h.
EXPORTS = ("moe_workspace_size", "moe_route", "moe_route_hash", "moe_bias_update", "moe_permute", "moe_expert_ffn",
           "moe_combine", "moe_layer_forward", "moe_route_static_scratch", "moe_quantize_fp8",
           "moe_ep_workspace_size", "moe_ep_layer_forward", "moe_ep_export_handle", "moe_ep_open_handle",
           "moe_ep_close_handle", "moe_sync_status", "moe_status_string")
MOE_STATIC_SCRATCH_BYTES = 8 << 20  # include/moe.h
MOE_EP_MAX_RANKS = 8
MOE_EP_HANDLE_BYTES = 72


class moe_config(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32), ("n_routed", ctypes.c_int32), ("n_shared", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
        ("moe_intermediate_size", ctypes.c_int32), ("score_fn", ctypes.c_int32),
        ("renormalize", ctypes.c_int32), ("routed_scaling_factor", ctypes.c_float),
        ("cap_policy", ctypes.c_int32), ("capacity_factor", ctypes.c_float), ("capacity", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down", "bias",
                 "w_gate_scale", "w_up_scale", "w_down_scale", "ws_gate_scale", "ws_up_scale", "ws_down_scale")]


class moe_diag(ctypes.Structure):
    _fields_ = [("overflowed", ctypes.c_int32), ("dropped", ctypes.c_int32), ("refined_tokens", ctypes.c_int32),
                ("max_load", ctypes.c_int32), ("refined_logits", ctypes.c_int32), ("status", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


class moe_ep_group(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("reserved", ctypes.c_int32), ("recv_rows", ctypes.c_int64),
                ("recv_x", ctypes.c_void_p * MOE_EP_MAX_RANKS), ("recv_out", ctypes.c_void_p * MOE_EP_MAX_RANKS),
                ("counts", ctypes.c_void_p * MOE_EP_MAX_RANKS), ("flags", ctypes.c_void_p * MOE_EP_MAX_RANKS)]


class moe_ep_rank(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("x", ctypes.c_void_p), ("weights", ctypes.POINTER(moe_weights)),
                ("y", ctypes.c_void_p), ("topk_idx_opt", ctypes.c_void_p), ("topk_w_opt", ctypes.c_void_p),
                ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t)]


DIAG_FIELDS = ("overflowed", "dropped", "refined_tokens", "max_load", "refined_logits", "status")

_P, _I64, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
_lib.moe_workspace_size.argtypes = [_P, _I64, ctypes.POINTER(ctypes.c_size_t)]
_lib.moe_route.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_permute.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_expert_ffn.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_combine.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_layer_forward.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_route_hash.argtypes = [_P, _I64, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_bias_update.argtypes = [_P, _P, _P, ctypes.c_float, _P]
_lib.moe_route_static_scratch.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _P, _P]
_lib.moe_quantize_fp8.argtypes = [_P, _I64, ctypes.c_int32, _P, _P, _P]
_lib.moe_ep_workspace_size.argtypes = [_P, ctypes.c_int32, _I64, _I64, ctypes.POINTER(ctypes.c_size_t)]
_lib.moe_ep_layer_forward.argtypes = [_P, _P, ctypes.c_int32, ctypes.c_int32, _P, _P]
_lib.moe_ep_export_handle.argtypes = [_P, _P]
_lib.moe_ep_open_handle.argtypes = [_P, ctypes.POINTER(ctypes.c_void_p)]
_lib.moe_ep_close_handle.argtypes = [_P]
_lib.moe_sync_status.argtypes = [_P, _P]
_lib.moe_status_string.argtypes = [ctypes.c_int]
_lib.moe_status_string.restype = ctypes.c_char_p
for _name in EXPORTS[:-1]:
    getattr(_lib, _name).restype = ctypes.c_int


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")
        self.status = status


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def make_config(d_model, n_routed, top_k, moe_intermediate_size, n_shared=0, n_group=1, topk_group=1,
                score_fn="softmax", renormalize=False, routed_scaling_factor=1.0, cap_policy="none",
                capacity_factor=0.0, capacity=0, dtype="bf16") -> moe_config:
    """A moe_config from the pages' field names (strings for the enums)."""
    return moe_config(
        d_model, n_routed, n_shared, top_k, n_group, topk_group, moe_intermediate_size,
        {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID, "sqrtsoftplus": MOE_SCORE_SQRTSOFTPLUS}[score_fn],
        int(bool(renormalize)),
        float(routed_scaling_factor),
        {"none": MOE_CAP_NONE, "overflow_next": MOE_CAP_OVERFLOW_NEXT, "drop": MOE_CAP_DROP}[cap_policy],
        float(capacity_factor), int(capacity), {"f32": MOE_F32, "bf16": MOE_BF16, "fp8": MOE_FP8}[dtype])


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream
    import torch

    return torch.cuda.current_stream().cuda_stream


def make_weights(w_router, w_gate, w_up, w_down, ws_gate=None, ws_up=None, ws_down=None, bias=None,
                 scales=None) -> moe_weights:
    """moe_weights from device tensors (the tensors must outlive every call that uses the struct).
    For MOE_FP8 the expert matrices are E4M3 codes (torch.uint8) and `scales` maps
    gate/up/down/ws_gate/ws_up/ws_down to their UE8M0 block-scale bytes."""
    sc = scales or {}
    return moe_weights(*(_ptr(t) for t in (w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, bias)),
                       *(_ptr(sc.get(k)) for k in ("gate", "up", "down", "ws_gate", "ws_up", "ws_down")))


def moe_workspace_size(cfg: moe_config, n: int) -> int:
    out = ctypes.c_size_t()
    _check(_lib.moe_workspace_size(ctypes.byref(cfg), n, ctypes.byref(out)), "moe_workspace_size")
    return out.value


def moe_route(cfg, n, x, weights, topk_idx, topk_w, expert_counts, diag, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(cfg), n, _ptr(x), ctypes.byref(weights), _ptr(topk_idx), _ptr(topk_w),
                          _ptr(expert_counts), _ptr(diag), _ptr(ws), ws.numel() * ws.element_size(),
                          _stream(stream)), "moe_route")


def moe_route_hash(cfg, n, x, token_ids, tid2eid, vocab, weights, topk_idx, topk_w, expert_counts, diag, ws,
                   stream=None):
    _check(_lib.moe_route_hash(ctypes.byref(cfg), n, _ptr(x), _ptr(token_ids), _ptr(tid2eid), vocab,
                               ctypes.byref(weights), _ptr(topk_idx), _ptr(topk_w), _ptr(expert_counts), _ptr(diag),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_route_hash")


def moe_bias_update(cfg, counts, bias, gamma, stream=None):
    _check(_lib.moe_bias_update(ctypes.byref(cfg), _ptr(counts), _ptr(bias), float(gamma), _stream(stream)),
           "moe_bias_update")


def moe_route_static_scratch(cfg, n, x, weights, topk_idx, topk_w, expert_counts, diag, stream=None):
    """moe_route without a workspace: the scratch is the library's static device array (see moe.h)."""
    _check(_lib.moe_route_static_scratch(ctypes.byref(cfg), n, _ptr(x), ctypes.byref(weights), _ptr(topk_idx),
                                         _ptr(topk_w), _ptr(expert_counts), _ptr(diag), _stream(stream)),
           "moe_route_static_scratch")


def moe_permute(cfg, n, x, topk_idx, offsets, perm_token, slot_dest, x_perm, ws, stream=None):
    _check(_lib.moe_permute(ctypes.byref(cfg), n, _ptr(x), _ptr(topk_idx), _ptr(offsets), _ptr(perm_token),
                            _ptr(slot_dest), _ptr(x_perm), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(stream)), "moe_permute")


def moe_expert_ffn(cfg, n, x_perm, offsets, weights, expert_out, ws, stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(cfg), n, _ptr(x_perm), _ptr(offsets), ctypes.byref(weights),
                               _ptr(expert_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_expert_ffn")


def moe_combine(cfg, n, expert_out, slot_dest, topk_w, x, weights, y, ws, stream=None):
    _check(_lib.moe_combine(ctypes.byref(cfg), n, _ptr(expert_out), _ptr(slot_dest), _ptr(topk_w), _ptr(x),
                            ctypes.byref(weights), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(stream)), "moe_combine")


def moe_layer_forward(cfg, n, x, weights, y, ws, topk_idx=None, topk_w=None, counts=None, diag=None, stream=None):
    _check(_lib.moe_layer_forward(ctypes.byref(cfg), n, _ptr(x), ctypes.byref(weights), _ptr(y), _ptr(topk_idx),
                                  _ptr(topk_w), _ptr(counts), _ptr(diag), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "moe_layer_forward")


def moe_quantize_fp8(x, codes, scale_bytes, stream=None):
    """E4M3 codes and UE8M0 scale bytes of bf16 rows x [rows, cols] in 1 x 128 tiles."""
    rows, cols = x.shape
    _check(_lib.moe_quantize_fp8(_ptr(x), rows, cols, _ptr(codes), _ptr(scale_bytes), _stream(stream)),
           "moe_quantize_fp8")


def moe_ep_recv_rows_bound(cfg, world, token_counts) -> int:
    """Rows an owner can receive at most: each token holds at most min(k, E / world) of its experts."""
    return max(1, int(sum(token_counts)) * min(cfg.top_k, cfg.n_routed // world))


def moe_ep_workspace_size(cfg, world, n, recv_rows) -> int:
    out = ctypes.c_size_t()
    _check(_lib.moe_ep_workspace_size(ctypes.byref(cfg), world, n, recv_rows, ctypes.byref(out)),
           "moe_ep_workspace_size")
    return out.value


def make_ep_group(recv_rows, recv_x, recv_out, counts, flags=None) -> moe_ep_group:
    """moe_ep_group from per-rank buffers: lists (one entry per rank) of device tensors or integer
    device addresses (peer mappings from ep_open_peers)."""
    world = len(recv_x)
    if not (1 <= world <= MOE_EP_MAX_RANKS) or not (len(recv_out) == len(counts) == world):
        raise ValueError("one recv_x, recv_out and counts buffer per rank, at most %d ranks" % MOE_EP_MAX_RANKS)

    def addr(v):
        return v if isinstance(v, int) or v is None else v.data_ptr()

    g = moe_ep_group()
    g.world, g.recv_rows = world, int(recv_rows)
    for q in range(world):
        g.recv_x[q], g.recv_out[q], g.counts[q] = addr(recv_x[q]), addr(recv_out[q]), addr(counts[q])
        g.flags[q] = addr(flags[q]) if flags is not None else None
    return g


def moe_ep_layer_forward(cfg, group, first_rank, ranks, stream=None):
    """One layer step of ranks first_rank .. first_rank + len(ranks) - 1. Each entry of `ranks` is a
    dict with n, x, weights (a moe_weights), y, ws and optionally topk_idx, topk_w."""
    arr = (moe_ep_rank * len(ranks))()
    keep = []
    for i, r in enumerate(ranks):
        w = r["weights"]
        keep.append(w)
        ws = r["ws"]
        arr[i] = moe_ep_rank(int(r["n"]), _ptr(r["x"]), ctypes.pointer(w), _ptr(r["y"]), _ptr(r.get("topk_idx")),
                             _ptr(r.get("topk_w")), _ptr(ws), ws.numel() * ws.element_size())
    _check(_lib.moe_ep_layer_forward(ctypes.byref(cfg), ctypes.byref(group), first_rank, len(ranks), arr,
                                     _stream(stream)), "moe_ep_layer_forward")


def moe_ep_export_handle(t) -> bytes:
    """Peer-mapping record (MOE_EP_HANDLE_BYTES bytes) of the device allocation holding tensor t."""
    buf = ctypes.create_string_buffer(MOE_EP_HANDLE_BYTES)
    _check(_lib.moe_ep_export_handle(_ptr(t), buf), "moe_ep_export_handle")
    return buf.raw


def moe_ep_open_handle(handle: bytes) -> int:
    if len(handle) != MOE_EP_HANDLE_BYTES:
        raise ValueError("a peer-mapping record has %d bytes" % MOE_EP_HANDLE_BYTES)
    out = ctypes.c_void_p()
    _check(_lib.moe_ep_open_handle(ctypes.create_string_buffer(handle, MOE_EP_HANDLE_BYTES), ctypes.byref(out)),
           "moe_ep_open_handle")
    return out.value


def moe_ep_close_handle(addr: int) -> None:
    _check(_lib.moe_ep_close_handle(addr), "moe_ep_close_handle")


def ep_open_peers(local: dict, rank: int, world: int, all_gather_object, export=None, open_=None) -> dict:
    """Exchange the peer-mapping records of this rank's exchange buffers with every rank of a
    process group and open the peers' buffers. `local` maps buffer names (recv_x, recv_out, counts,
    flags) to this rank's tensors; `all_gather_object(obj)` returns the list of every rank's obj
    (e.g. a wrapper of torch.distributed.all_gather_object). Returns name -> per-rank list with
    this rank's tensor at `rank` and the peers' mapped addresses elsewhere; release those with
    moe_ep_close_handle."""
    export = export or moe_ep_export_handle
    open_ = open_ or moe_ep_open_handle
    mine = {k: export(t) for k, t in local.items()}
    records = all_gather_object(mine)
    if len(records) != world:
        raise RuntimeError("expected %d records, got %d" % (world, len(records)))
    return {k: [t if q == rank else open_(records[q][k]) for q in range(world)] for k, t in local.items()}


def moe_sync_status(ws, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word of the workspace."""
    return _lib.moe_sync_status(_ptr(ws), _stream(stream))


def lib_handle():
    return _lib
