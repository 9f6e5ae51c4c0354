"""ctypes bindings of the host fill (``libsynth.so``) and the device fill
(``libsynth_cuda.so``) of the counter-based generator defined in ``synth.h``."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynth.so")
CUDA_LIB = os.path.join(_HERE, "libsynth_cuda.so")

NORMAL, UNIFORM, TERNARY, BYTE, SIGNED_CODE = 0, 1, 2, 3, 4
STREAM = dict(x=1, w_r=2, bias=3, w_gate=4, w_up=5, w_down=6, ws_gate=7, ws_up=8, ws_down=9,
              w_gate_q=10, w_up_q=11, w_down_q=12, ws_gate_q=13, ws_up_q=14, ws_down_q=15,
              w_gate_s=16, w_up_s=17, w_down_s=18, ws_gate_s=19, ws_up_s=20, ws_down_s=21)


def _stale(out, *srcs):
    return not os.path.exists(out) or os.path.getmtime(out) < max(os.path.getmtime(s) for s in srcs)


def build_host(force=False):
    src, hdr = os.path.join(_HERE, "synth_host.c"), os.path.join(_HERE, "synth.h")
    if force or _stale(HOST_LIB, src, hdr):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                               "-shared", "-o", HOST_LIB, src])
    return HOST_LIB


def build_cuda(force=False):
    src, hdr = os.path.join(_HERE, "synth_cuda.cu"), os.path.join(_HERE, "synth.h")
    if force or _stale(CUDA_LIB, src, hdr):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                               "-fmad=false", "-Xcompiler", "-fPIC", "-shared", "-o", CUDA_LIB, src])
    return CUDA_LIB


_host = None
_cuda = None


def _host_lib():
    global _host
    if _host is None:
        _host = ctypes.CDLL(build_host())
        args = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                ctypes.c_int, ctypes.c_double, ctypes.c_double]
        _host.synth_fill_f32.argtypes = args
        _host.synth_fill_bf16.argtypes = args
        _host.synth_fill_u8.argtypes = args
    return _host


def _cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(CUDA_LIB):
            raise RuntimeError(f"{CUDA_LIB} is missing: run __graft_entry__.build() first")
        _cuda = ctypes.CDLL(CUDA_LIB)
        _cuda.synth_cuda_fill.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_double, ctypes.c_void_p]
        _cuda.synth_cuda_fill.restype = ctypes.c_int
    return _cuda


def host(shape, dtype: str, seed: int, stream: int, kind: int, a: float, b: float = 0.0,
         start: int = 0) -> np.ndarray:
    """Elements [start, start + prod(shape)) of a stream, as float32, raw bf16 bits (uint16) or bytes ("u8")."""
    count = int(np.prod(shape))
    if dtype == "f32":
        out = np.empty(count, np.float32)
        _host_lib().synth_fill_f32(out.ctypes.data, count, seed, stream, start, kind, a, b)
    elif dtype == "bf16":
        out = np.empty(count, np.uint16)
        _host_lib().synth_fill_bf16(out.ctypes.data, count, seed, stream, start, kind, a, b)
    elif dtype == "u8":
        out = np.empty(count, np.uint8)
        _host_lib().synth_fill_u8(out.ctypes.data, count, seed, stream, start, kind, a, b)
    else:
        raise ValueError(dtype)
    return out.reshape(shape)


def device(t, seed: int, stream: int, kind: int, a: float, b: float = 0.0, start: int = 0):
    """Fill a contiguous CUDA tensor (torch.float32, torch.bfloat16 or torch.uint8) in place on its current stream."""
    import torch

    assert t.is_cuda and t.is_contiguous()
    dt = {torch.float32: 0, torch.bfloat16: 1, torch.uint8: 2}[t.dtype]
    s = torch.cuda.current_stream(t.device).cuda_stream
    rc = _cuda_lib().synth_cuda_fill(t.data_ptr(), dt, t.numel(), seed, stream, start, kind, a, b, s)
    if rc != 0:
        raise RuntimeError(f"synth_cuda_fill failed with cudaError {rc}")
    return t
