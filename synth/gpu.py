"""Draws the seeded inputs directly on the GPU (bit-identical to synth.workloads).

Used for workloads too large to draw on the host (the 131072-key decode cache
holds 17 GB of bf16).  Test-support code: no attention arithmetic here.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

from . import workloads as sw

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libsynth_gen.so")
SRC = os.path.join(_HERE, "csrc", "synth_gen.cu")

KIND = {torch.float64: 0, torch.float32: 1, torch.bfloat16: 2}

_lib = None


def build(force: bool = False) -> str:
    """nvcc for sm_100a with fused multiply-add contraction disabled."""
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC):
        return LIB_PATH
    os.makedirs(os.path.dirname(LIB_PATH), exist_ok=True)
    tmp = LIB_PATH + ".tmp"
    subprocess.run(["nvcc", "-shared", "-Xcompiler", "-fPIC", "-O3", "-fmad=false", "-std=c++17",
                    "-gencode", "arch=compute_100a,code=sm_100a", SRC, "-o", tmp], check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} missing: run synth.gpu.build()")
        lib = ctypes.CDLL(LIB_PATH)
        lib.synth_normal.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_ulonglong,
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_void_p]
        lib.synth_normal.restype = ctypes.c_int
        _lib = lib
    return _lib


_COEF = None


def _coef():
    global _COEF
    if _COEF is None:
        _COEF = tuple(np.ascontiguousarray(a, dtype=np.float64) for a in (sw.LOG_COEF, sw.COS_COEF, sw.SIN_COEF))
    return _COEF


def normal_into(dst: torch.Tensor, key: int, start: int = 0):
    """Fills contiguous CUDA tensor `dst` with elements [start, start+numel) of stream `key`."""
    assert dst.is_cuda and dst.is_contiguous() and dst.dtype in KIND
    lc, cc, sc = _coef()
    st = _load().synth_normal(ctypes.c_void_p(dst.data_ptr()), int(start), int(dst.numel()), ctypes.c_ulonglong(key),
                              KIND[dst.dtype], lc.ctypes.data, cc.ctypes.data, sc.ctypes.data, sw.LN2,
                              sw.HALF_PI, sw.SQRT_HALF,
                              ctypes.c_void_p(torch.cuda.current_stream(dst.device).cuda_stream))
    if st != 0:
        raise RuntimeError(f"synth_normal failed ({st})")
    return dst


def _torch_dtype(r: sw.Recipe):
    return torch.bfloat16 if r.dtype == "bf16" else torch.float32


def _host_to_device(arr: np.ndarray, r: sw.Recipe, device) -> torch.Tensor:
    if r.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def generate_on_device(r: sw.Recipe, device="cuda") -> dict:
    """q, k, v, sink, bias of recipe r as CUDA tensors (same bits as synth.workloads.generate)."""
    out = {}
    if sw.gpu_drawable(r):
        streams = {"q": sw.STREAM_Q, "k": sw.STREAM_K, "v": sw.STREAM_V}
        for t, shp in sw.shapes(r).items():
            x = torch.empty(shp, dtype=_torch_dtype(r), device=device)
            normal_into(x, sw.stream_key(r.seed, streams[t]))
            out[t] = x
    else:
        host = sw.generate(r)
        for t in ("q", "k", "v"):
            out[t] = _host_to_device(host[t], r, device)
    s = sw.sink_logits(r)
    out["sink"] = None if s is None else torch.from_numpy(s).to(device)
    b = sw.bias_matrix(r)
    out["bias"] = None if b is None else torch.from_numpy(b).to(device)
    ki = sw.key_index_set(r)
    out["key_idx"] = None if ki is None else torch.from_numpy(ki).to(device)
    km = sw.keep_matrix(r)
    out["mask_bits"] = None if km is None else torch.from_numpy(sw.pack_mask_bits(km).view(np.int32)).to(device)
    ks, ke = sw.kv_ranges(r)
    out["kv_start"] = None if ks is None else torch.from_numpy(ks).to(device)
    out["kv_end"] = None if ke is None else torch.from_numpy(ke).to(device)
    return out


def to_device(arr: np.ndarray, r: sw.Recipe, device="cuda") -> torch.Tensor:
    return _host_to_device(arr, r, device)
