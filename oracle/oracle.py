"""ctypes binding of the fp64 CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code with
the CUDA library. Tensors are numpy arrays; bf16 tensors are ``uint16`` arrays
holding the raw bf16 bits, binary32 tensors are ``float32`` arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` with gcc into ``oracle/liboracle.so``."""
    src = os.path.join(_HERE, "moe_oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "moe_oracle.h"))
    ):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, src, "-lm"]
        )
    return _LIB_PATH


class OracleCfg(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32),
        ("n_routed", ctypes.c_int32),
        ("n_shared", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("n_group", ctypes.c_int32),
        ("topk_group", ctypes.c_int32),
        ("inter", ctypes.c_int32),
        ("score_fn", ctypes.c_int32),
        ("renormalize", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_double),
        ("cap_policy", ctypes.c_int32),
        ("capacity_factor", ctypes.c_double),
        ("capacity", ctypes.c_int32),
    ]


class OracleStats(ctypes.Structure):
    _fields_ = [
        ("overflowed", ctypes.c_int64),
        ("dropped", ctypes.c_int64),
        ("exempt_tokens", ctypes.c_int64),
        ("capacity", ctypes.c_int64),
    ]


class DsArch(ctypes.Structure):
    _fields_ = [
        (name, ctypes.c_int64)
        for name in (
            "n_layers d_model q_lora_rank kv_lora_rank n_heads qk_nope_dim qk_rope_dim v_head_dim "
            "vocab first_k_dense dense_inter n_routed n_shared top_k moe_inter"
        ).split()
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        _lib.oracle_router_logits.argtypes = [i64, i32, i32, P, i32, P, i32, P]
        _lib.oracle_route.argtypes = [P, i64, P, P, P, P, P, P, P]
        _lib.oracle_route_capacity.argtypes = [P, i64, P, P, P, P, P, P]
        _lib.oracle_capacity_value.argtypes = [P, i64]
        _lib.oracle_capacity_value.restype = i64
        _lib.oracle_dispatch.argtypes = [i64, i32, i32, P, P, P, P, P]
        _lib.oracle_dispatch.restype = i64
        _lib.oracle_swiglu.argtypes = [i32, i32, i64, P, P, P, P, i32, P]
        _lib.oracle_combine.argtypes = [i64, i32, i32, P, P, P, P, P]
        _lib.oracle_layer.argtypes = [P, i64] + [P] * 9 + [i32] + [P] * 6
        _lib.oracle_ds_params.argtypes = [P, P, P]
        _lib.oracle_route_hash.argtypes = [P, i64, P, P, P, P, P]
        _lib.oracle_bias_update.argtypes = [i32, P, P, ctypes.c_double, P]
        _lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_value.restype = ctypes.c_double
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_ue8m0_exponent.argtypes = [ctypes.c_double]
        _lib.oracle_ue8m0_exponent.restype = i32
        _lib.oracle_quantize_rows.argtypes = [i64, i32, P, i32, P, P]
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    raise TypeError(f"oracle tensors are float32 or uint16 (bf16 bits), got {a.dtype}")


def _c(a, dtype=None):
    if a is None:
        return None
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


@dataclass
class Cfg:
    """Layer configuration in the pages' field names."""

    d_model: int
    n_routed: int
    top_k: int
    moe_intermediate_size: int
    n_shared: int = 0
    n_group: int = 1
    topk_group: int = 1
    score_fn: str = "softmax"  # or "sigmoid", "sqrtsoftplus"
    renormalize: bool = False
    routed_scaling_factor: float = 1.0
    cap_policy: str = "none"  # "none" | "overflow_next" | "drop"
    capacity_factor: float = 0.0
    capacity: int = 0

    def c(self) -> OracleCfg:
        return OracleCfg(
            self.d_model,
            self.n_routed,
            self.n_shared,
            self.top_k,
            self.n_group,
            self.topk_group,
            self.moe_intermediate_size,
            {"softmax": 0, "sigmoid": 1, "sqrtsoftplus": 2}[self.score_fn],
            int(bool(self.renormalize)),
            float(self.routed_scaling_factor),
            {"none": 0, "overflow_next": 1, "drop": 2}[self.cap_policy],
            float(self.capacity_factor),
            int(self.capacity),
        )


def router_logits(x: np.ndarray, w_r: np.ndarray) -> np.ndarray:
    x, w_r = _c(x), _c(w_r)
    n, d = x.shape
    E = w_r.shape[0]
    out = np.empty((n, E), np.float64)
    lib().oracle_router_logits(n, d, E, _ptr(x), _dt(x), _ptr(w_r), _dt(w_r), _ptr(out))
    return out


def route(cfg: Cfg, logits: np.ndarray, bias=None, want_ranking=False):
    """Routing without capacity. Returns (topk_idx, topk_w, exempt, ranking|None, stats)."""
    logits = _c(logits, np.float64)
    bias = _c(bias, np.float32)
    n = logits.shape[0]
    k, E = cfg.top_k, cfg.n_routed
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    ex = np.empty(n, np.uint8)
    rk = np.empty((n, E), np.int32) if want_ranking else None
    st = OracleStats()
    c = cfg.c()
    lib().oracle_route(
        ctypes.byref(c), n, _ptr(logits), _ptr(bias), _ptr(idx), _ptr(w), _ptr(ex), _ptr(rk),
        ctypes.byref(st),
    )
    return idx, w, ex.astype(bool), rk, st


def route_capacity(cfg: Cfg, logits: np.ndarray, bias=None):
    """Routing with the configured capacity policy. Returns (topk_idx, topk_w, exempt, stats)."""
    logits = _c(logits, np.float64)
    bias = _c(bias, np.float32)
    n = logits.shape[0]
    k = cfg.top_k
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    ex = np.empty(n, np.uint8)
    st = OracleStats()
    c = cfg.c()
    lib().oracle_route_capacity(
        ctypes.byref(c), n, _ptr(logits), _ptr(bias), _ptr(idx), _ptr(w), _ptr(ex), ctypes.byref(st)
    )
    return idx, w, ex.astype(bool), st


def route_hash(cfg: Cfg, logits: np.ndarray, token_ids: np.ndarray, tid2eid: np.ndarray):
    """Hash routing: (topk_idx, topk_w)."""
    logits = _c(logits, np.float64)
    token_ids = _c(token_ids, np.int32)
    tid2eid = _c(tid2eid, np.int32)
    n = logits.shape[0]
    idx = np.empty((n, cfg.top_k), np.int32)
    w = np.empty((n, cfg.top_k), np.float64)
    c = cfg.c()
    lib().oracle_route_hash(ctypes.byref(c), n, _ptr(logits), _ptr(token_ids), _ptr(tid2eid), _ptr(idx), _ptr(w))
    return idx, w


def bias_update(counts: np.ndarray, bias: np.ndarray, gamma: float) -> np.ndarray:
    counts = _c(counts, np.int32)
    bias = _c(bias, np.float32)
    out = np.empty(len(counts), np.float64)
    lib().oracle_bias_update(len(counts), _ptr(counts), _ptr(bias), gamma, _ptr(out))
    return out


def capacity_value(cfg: Cfg, n: int) -> int:
    c = cfg.c()
    return int(lib().oracle_capacity_value(ctypes.byref(c), n))


def dispatch(topk_idx: np.ndarray, E: int):
    """Returns (counts[E], offsets[E+1], perm_token[kept], slot_dest[n,k])."""
    topk_idx = _c(topk_idx, np.int32)
    n, k = topk_idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(max(n * k, 1), np.int32)
    dest = np.empty((n, k), np.int32)
    kept = lib().oracle_dispatch(n, k, E, _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(dest))
    return counts, offsets, perm[:kept].copy(), dest


def swiglu(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """x[m, d] (float64) through one SwiGLU expert with W_g, W_u [I, d], W_d [d, I]."""
    x = _c(x, np.float64)
    w_gate, w_up, w_down = _c(w_gate), _c(w_up), _c(w_down)
    assert w_gate.dtype == w_up.dtype == w_down.dtype
    m, d = x.shape
    I = w_gate.shape[0]
    out = np.empty((m, d), np.float64)
    lib().oracle_swiglu(d, I, m, _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _dt(w_gate), _ptr(out))
    return out


def combine(eo: np.ndarray, slot_dest: np.ndarray, topk_w: np.ndarray, sh=None) -> np.ndarray:
    eo = _c(eo, np.float64)
    slot_dest = _c(slot_dest, np.int32)
    topk_w = _c(topk_w, np.float64)
    sh = _c(sh, np.float64)
    n, k = slot_dest.shape
    d = eo.shape[1]
    y = np.empty((n, d), np.float64)
    lib().oracle_combine(n, k, d, _ptr(eo), _ptr(slot_dest), _ptr(topk_w), _ptr(sh), _ptr(y))
    return y


def layer(cfg: Cfg, x, w_r, w_gate, w_up, w_down, bias=None, ws_gate=None, ws_up=None, ws_down=None):
    """Whole layer. Returns dict(y, topk_idx, topk_w, counts, exempt, stats)."""
    x, w_r, w_gate, w_up, w_down = (_c(a) for a in (x, w_r, w_gate, w_up, w_down))
    ws_gate, ws_up, ws_down = (_c(a) for a in (ws_gate, ws_up, ws_down))
    bias = _c(bias, np.float32)
    dt = _dt(x)
    for a in (w_r, w_gate, w_up, w_down, ws_gate, ws_up, ws_down):
        assert a is None or _dt(a) == dt
    n = x.shape[0]
    k, E, d = cfg.top_k, cfg.n_routed, cfg.d_model
    y = np.empty((n, d), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    counts = np.empty(E, np.int32)
    ex = np.empty(n, np.uint8)
    st = OracleStats()
    c = cfg.c()
    lib().oracle_layer(
        ctypes.byref(c), n, _ptr(x), _ptr(w_r), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), dt, _ptr(y), _ptr(idx), _ptr(w), _ptr(counts),
        _ptr(ex), ctypes.byref(st),
    )
    return dict(y=y, topk_idx=idx, topk_w=w, counts=counts, exempt=ex.astype(bool), stats=st)


def ds_params(**fields) -> tuple[int, int]:
    a = DsArch(**fields)
    total, active = ctypes.c_int64(), ctypes.c_int64()
    lib().oracle_ds_params(ctypes.byref(a), ctypes.byref(total), ctypes.byref(active))
    return total.value, active.value


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits (uint16) or float32 to float64 (input decoding only)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ---- FP8 experts (page "15. DeepSeek: MLA, MoE and MTP", FP8 section) -------------------------
# E4M3 matrix inputs with one UE8M0 scale (2^(byte - 127)) per 1 x 128 activation tile and per
# 128 x 128 weight block. The layer below quantises activations (x, and h between the two expert
# matrices) exactly as defined by oracle_quantize_rows and multiplies the dequantised values in
# binary64 (each dequantised value is exact: a 4-bit significand times a power of two).

def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(v))


def ue8m0_exponent(amax: float) -> int:
    return lib().oracle_ue8m0_exponent(float(amax))


def e4m3_table() -> np.ndarray:
    """binary64 value of every code 0..255 (NaN for the two NaN codes)."""
    return np.array([lib().oracle_e4m3_value(c) for c in range(256)], np.float64)


def quantize_rows(a: np.ndarray):
    """Rows of a [rows, cols] (binary64, binary32 or bf16 bits) in 1 x 128 tiles -> (codes uint8, scale bytes uint8)."""
    a = _c(a)
    if a.dtype == np.float64:
        dt = 2
    else:
        dt = _dt(a)
    rows, cols = a.shape
    assert cols % 128 == 0
    codes = np.empty((rows, cols), np.uint8)
    sb = np.empty((rows, cols // 128), np.uint8)
    lib().oracle_quantize_rows(rows, cols, _ptr(a), dt, _ptr(codes), _ptr(sb))
    return codes, sb


def dequant_rows(codes: np.ndarray, scale_bytes: np.ndarray) -> np.ndarray:
    """codes [rows, cols] with one scale byte per 1 x 128 tile -> binary64."""
    v = e4m3_table()[codes]
    s = np.ldexp(1.0, scale_bytes.astype(np.int32) - 127)
    return v * np.repeat(s, 128, axis=1)


def dequant_blocks(codes: np.ndarray, scale_bytes: np.ndarray) -> np.ndarray:
    """Weight codes [N, K] with one scale byte per 128 x 128 block [ceil(N/128), K/128] -> binary64."""
    N, K = codes.shape
    v = e4m3_table()[codes]
    s = np.ldexp(1.0, scale_bytes.astype(np.int32) - 127)
    s = np.repeat(np.repeat(s, 128, axis=0)[:N], 128, axis=1)[:, :K]
    return v * s


def round_to_bf16(a64: np.ndarray) -> np.ndarray:
    """binary64 -> bf16, one rounding to nearest with ties to even, widened back to binary64.

    bf16 keeps 8 significant bits with binary32's exponent range, so a value in [2^(e-1), 2^e)
    lands on the grid 2^(e-8); below the smallest normal (2^-126) the grid stays 2^-133
    (subnormals). Magnitudes that round past the largest finite bf16 become infinite."""
    a64 = np.asarray(a64, np.float64)
    _, e = np.frexp(a64)
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)
    r = np.rint(a64 / q) * q  # the division and product are exact (powers of two); rint ties to even
    big = np.abs(r) >= 2.0 ** 128
    return np.where(big, np.copysign(np.inf, a64), r)


def swiglu_fp8(x64: np.ndarray, wg, wu, wd) -> np.ndarray:
    """One FP8 expert on rows x64 [m, d]: quantise x, gate/up with dequantised weights, SwiGLU,
    quantise h, down. wg/wu/wd are (codes, scale bytes) pairs. h is an activation of the layer,
    held in the layer's activation type (bf16, like x and y) when it enters the down matrix, so
    its E4M3 codes are decided on h rounded once from binary64 to bf16 (an E4M3 step is 2^4 bf16
    steps, so deciding the codes from binary64 h instead moves about 1 in 64 codes by one E4M3
    step)."""
    xq, xs = quantize_rows(x64)
    xd = dequant_rows(xq, xs)
    g = xd @ dequant_blocks(*wg).T
    u = xd @ dequant_blocks(*wu).T
    h = round_to_bf16(g / (1.0 + np.exp(-g)) * u)
    hq, hs = quantize_rows(h)
    return dequant_rows(hq, hs) @ dequant_blocks(*wd).T


def layer_fp8(cfg: Cfg, x, w_r, bias, w8: dict, ws8: dict = None):
    """Whole layer with FP8 experts. x, w_r are bf16 bits (routing as in layer()); w8 holds
    gate/up/down as (codes [E, N, K], scale bytes [E, N/128, K/128]); ws8 the shared experts'
    (codes [N, K], scale bytes). Returns dict(y, topk_idx, topk_w, counts, exempt, stats)."""
    lg = router_logits(x, w_r)
    idx, w, ex, st = route_capacity(cfg, lg, bias)
    counts, offsets, perm, dest = dispatch(idx, cfg.n_routed)
    x64 = bf16_to_f64(x)
    eo = np.zeros((max(len(perm), 1), cfg.d_model), np.float64)
    for e in range(cfg.n_routed):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            eo[lo:hi] = swiglu_fp8(x64[perm[lo:hi]], (w8["gate"][0][e], w8["gate"][1][e]),
                                   (w8["up"][0][e], w8["up"][1][e]), (w8["down"][0][e], w8["down"][1][e]))
    sh = None
    if ws8 is not None:
        sh = swiglu_fp8(x64, ws8["gate"], ws8["up"], ws8["down"])
    y = combine(eo, dest, w, sh)
    return dict(y=y, topk_idx=idx, topk_w=w, counts=counts, exempt=ex, stats=st)


def ep_recv_layout(topk_idx_per_rank, E: int, world: int):
    """Rows each owner receives when `world` ranks share a layer and rank q owns experts
    [q E/world, (q+1) E/world) (page "15. DeepSeek: MLA, MoE and MTP", section "V3 MoE": one
    expert group per node). Order at an owner: its experts ascending; inside an expert the source
    ranks ascending; inside a source its tokens ascending. Returns, per owner q, (rows, offsets):
    rows [m, 2] = (source rank, source token) of each received row, offsets [E/world + 1] the row
    range of each owned expert."""
    Eq = E // world
    out = []
    for q in range(world):
        rows, offsets = [], [0]
        for e in range(q * Eq, (q + 1) * Eq):
            for s, idx in enumerate(topk_idx_per_rank):
                toks = np.nonzero((np.asarray(idx) == e).any(axis=1))[0]
                rows.extend((s, int(t)) for t in toks)
            offsets.append(len(rows))
        out.append((np.asarray(rows, np.int64).reshape(-1, 2), np.asarray(offsets, np.int64)))
    return out
