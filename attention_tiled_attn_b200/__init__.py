"""Fused attention forward for NVIDIA B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI declared in ``include/attn_b200.h``.  It only
marshals arguments (shapes, dtypes, data pointers, the current CUDA stream);
every step of the computation runs in the library's CUDA kernels.  There is
no CPU fallback: without the built library or a CUDA device the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libattn_b200.so")

MODES = {"dot": 0, "rbf": 1, "sink": 2}
MASKS = {"none": 0, "causal": 1, "window": 2}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}

ATTN_OK = 0


class AttnError(RuntimeError):
    """A non-zero status returned by the library."""

    def __init__(self, status: int, text: str):
        super().__init__(f"attn status {status}: {text}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library not built: {path} is missing (run python -m attention_tiled_attn_b200.build)")
    lib = ctypes.CDLL(path)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp, ci, ci, vp, ci, vp]
    lib.attn_fwd.restype = ci
    lib.attn_fwd_streaming.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp, ci, ci, vp, ci, vp]
    lib.attn_fwd_streaming.restype = ci
    lib.attn_decode_indexed.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci, cf, vp, ci, ci, vp,
                                        vp]
    lib.attn_decode_indexed.restype = ci
    lib.attn_fwd_padded.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp, ci, ci, vp, vp, vp, ci,
                                    vp]
    lib.attn_fwd_padded.restype = ci
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp, ci, ci, ci,
                             vp, vp, vp, vp]
    lib.attn_bwd.restype = ci
    lib.attn_status_string.argtypes = [ci]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_release_workspace.argtypes = []
    lib.attn_release_workspace.restype = None
    lib.attn_device_status.argtypes = [vp]
    lib.attn_device_status.restype = ci
    lib.attn_version.argtypes = []
    lib.attn_version.restype = ci
    lib.attn_exp2_poly_eval.argtypes = [vp, vp, ci, vp]
    lib.attn_exp2_poly_eval.restype = ci
    lib.attn_decode_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp, ci, ci, vp, vp]
    lib.attn_decode_fwd_noalloc.restype = ci
    lib.attn_test_wait_timeout.argtypes = [ci, vp]
    lib.attn_test_wait_timeout.restype = ci
    lib.attn_test_fail_workspace_allocs.argtypes = [ci]
    lib.attn_test_fail_workspace_allocs.restype = ci
    lib.attn_decode_noalloc_scratch_bytes.argtypes = []
    lib.attn_decode_noalloc_scratch_bytes.restype = ctypes.c_size_t
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()


def _check(status: int):
    if status != ATTN_OK:
        raise AttnError(status, status_string(status))


def _check_kinds(mode: str, mask_kind: str, keep_first: int = 0, masks=None):
    """Rejects an unknown mode or mask kind, and kept keys without the streaming mask."""
    if mode not in MODES:
        raise ValueError(f"unknown mode {mode!r}")
    if mask_kind not in (masks or (*MASKS, "streaming")):
        raise ValueError(f"unknown mask kind {mask_kind!r}")
    if int(keep_first) != 0 and mask_kind != "streaming":
        raise ValueError("keep_first needs mask_kind 'streaming'")


def _same_device(ref: torch.Tensor, **tensors):
    """The library reads every pointer on ref's device; a tensor elsewhere is rejected."""
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, not on {ref.device} with q")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def attn_fwd_raw(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, N, Hq, H, L, S, E, Ev, scale, mode, sink_ptr,
                 mask_kind, window, bias_ptr, dtype, stream_ptr) -> int:
    """The C entry point with integer pointers; returns the status code."""
    lib = load_library()
    c = lambda p: None if p is None else ctypes.c_void_p(int(p))  # noqa: E731
    return lib.attn_fwd(c(q_ptr), c(k_ptr), c(v_ptr), c(out_ptr), c(lse_ptr), int(N), int(Hq), int(H), int(L),
                        int(S), int(E), int(Ev), float(scale), int(mode), c(sink_ptr), int(mask_kind),
                        int(window), c(bias_ptr), int(dtype), c(stream_ptr))


def attn_bwd_raw(q_ptr, k_ptr, v_ptr, out_ptr, dout_ptr, lse_ptr, dq_ptr, dk_ptr, dv_ptr, dsink_ptr, N, Hq, H, L, S,
                 E, Ev, scale, mode, sink_ptr, mask_kind, window, stream_ptr, keep_first=0, bits_ptr=None,
                 start_ptr=None, end_ptr=None) -> int:
    """The backward C entry point with integer pointers; returns the status code."""
    lib = load_library()
    c = lambda p: None if p is None else ctypes.c_void_p(int(p))  # noqa: E731
    return lib.attn_bwd(c(q_ptr), c(k_ptr), c(v_ptr), c(out_ptr), c(dout_ptr), c(lse_ptr), c(dq_ptr), c(dk_ptr),
                        c(dv_ptr), c(dsink_ptr), int(N), int(Hq), int(H), int(L), int(S), int(E), int(Ev),
                        float(scale), int(mode), c(sink_ptr), int(mask_kind), int(window), int(keep_first),
                        c(bits_ptr), c(start_ptr), c(end_ptr), c(stream_ptr))


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
             dout: torch.Tensor, *, scale: float, mode: str = "dot", sink: torch.Tensor | None = None,
             mask_kind: str = "none", window: int = 0, stream: torch.cuda.Stream | None = None, keep_first: int = 0,
             mask_bits: torch.Tensor | None = None, kv_start: torch.Tensor | None = None,
             kv_end: torch.Tensor | None = None):
    """Gradients (dq, dk, dv, dsink) of attn_fwd's output; float32 tensors, dsink None without a sink.

    q, k, v, out, dout: contiguous bfloat16 CUDA tensors (the forward's inputs and
    output, and the loss gradient of the output); lse: the forward's float32 lse.
    mask_kind "streaming" with window and keep_first, and mask_bits / kv_start /
    kv_end, mirror attn_fwd's arguments.
    """
    _check_kinds(mode, mask_kind, keep_first)
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D bfloat16 CUDA tensor")
    N, Hq, L, E = q.shape
    _, H, S, _ = k.shape
    Ev = v.shape[3]
    if tuple(out.shape) != (N, Hq, L, Ev) or tuple(dout.shape) != (N, Hq, L, Ev):
        raise ValueError("out and dout must be (N, Hq, L, Ev)")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (N, Hq, L) or not lse.is_cuda or not lse.is_contiguous():
        raise ValueError("lse must be the forward's float32 (N, Hq, L) tensor")
    if sink is not None and (sink.dtype != torch.float32 or sink.numel() != Hq or not sink.is_cuda
                             or not sink.is_contiguous()):
        raise ValueError("sink must be a contiguous CUDA float32 tensor of Hq values")
    for name, t, shape in (("mask_bits", mask_bits, (L, (S + 31) // 32)), ("kv_start", kv_start, (N,)),
                           ("kv_end", kv_end, (N,))):
        if t is not None and (not t.is_cuda or t.dtype != torch.int32 or tuple(t.shape) != shape
                              or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA int32 tensor of shape {shape}")
    _same_device(q, k=k, v=v, out=out, lse=lse, dout=dout, sink=sink, mask_bits=mask_bits, kv_start=kv_start,
                 kv_end=kv_end)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    dsink = torch.empty(Hq, dtype=torch.float32, device=q.device) if sink is not None else None
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    if mask_kind == "streaming":
        kind, keep = MASKS["window"], int(keep_first)
    else:
        kind, keep = MASKS[mask_kind], 0
    with torch.cuda.device(q.device):
        st = load_library().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                     _ptr(dv), _ptr(dsink), N, Hq, H, L, S, E, Ev, float(scale), MODES[mode],
                                     _ptr(sink), kind, int(window), keep, _ptr(mask_bits), _ptr(kv_start),
                                     _ptr(kv_end), ctypes.c_void_p(stream.cuda_stream))
    _check(st)
    return dq, dk, dv, dsink


def attn_fwd_padded_raw(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, N, Hq, H, L, S, E, Ev, scale, mode, sink_ptr,
                        mask_kind, window, bits_ptr, start_ptr, end_ptr, dtype, stream_ptr) -> int:
    """The keep-bits / key-padding C entry point with integer pointers; returns the status code."""
    lib = load_library()
    c = lambda p: None if p is None else ctypes.c_void_p(int(p))  # noqa: E731
    return lib.attn_fwd_padded(c(q_ptr), c(k_ptr), c(v_ptr), c(out_ptr), c(lse_ptr), int(N), int(Hq), int(H), int(L),
                               int(S), int(E), int(Ev), float(scale), int(mode), c(sink_ptr), int(mask_kind),
                               int(window), c(bits_ptr), c(start_ptr), c(end_ptr), int(dtype), c(stream_ptr))


def attn_fwd_streaming_raw(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, N, Hq, H, L, S, E, Ev, scale, mode, sink_ptr,
                           window, keep_first, bias_ptr, dtype, stream_ptr) -> int:
    """The streaming-mask C entry point with integer pointers; returns the status code."""
    lib = load_library()
    c = lambda p: None if p is None else ctypes.c_void_p(int(p))  # noqa: E731
    return lib.attn_fwd_streaming(c(q_ptr), c(k_ptr), c(v_ptr), c(out_ptr), c(lse_ptr), int(N), int(Hq), int(H),
                                  int(L), int(S), int(E), int(Ev), float(scale), int(mode), c(sink_ptr),
                                  int(window), int(keep_first), c(bias_ptr), int(dtype), c(stream_ptr))


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: float, mode: str = "dot",
             sink: torch.Tensor | None = None, mask_kind: str = "none", window: int = 0,
             bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None, keep_first: int = 0,
             mask_bits: torch.Tensor | None = None, kv_start: torch.Tensor | None = None,
             kv_end: torch.Tensor | None = None):
    """out = softmax(z + B) V on the GPU.  Returns (out, lse).

    q (N, Hq, L, E), k (N, H, S, E), v (N, H, S, Ev): contiguous CUDA tensors,
    all bfloat16 or all float32.  sink: (Hq,) float32 or None.  bias: (L, S)
    float32 or None.  mode: "dot", "rbf" or "sink"; mask_kind: "none",
    "causal", "window" or "streaming" (the first ``keep_first`` keys plus the
    last ``window`` keys, through attn_fwd_streaming).  out/lse may be given
    (contiguous, right shape).  mask_bits (L, ceil(S/32)) int32 (bit j%32 of
    word j/32 set: row may attend key j), kv_start / kv_end (N,) int32 key
    padding: any of them routes the call through attn_fwd_padded (no bias).
    """
    _check_kinds(mode, mask_kind, keep_first)
    load_library()
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-D tensor")
    if q.dtype not in DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype bfloat16 or float32")
    N, Hq, L, E = q.shape
    Nk, H, S, Ek = k.shape
    Nv, Hv, Sv, Ev = v.shape
    if Nk != N or Nv != N or Hv != H or Sv != S or Ek != E:
        raise ValueError("inconsistent q/k/v shapes")
    if sink is not None and (sink.dtype != torch.float32 or sink.numel() != Hq or not sink.is_cuda
                             or not sink.is_contiguous()):
        raise ValueError("sink must be a contiguous CUDA float32 tensor of Hq values")
    if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (L, S) or not bias.is_cuda
                             or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous CUDA float32 (L, S) tensor")
    if out is None:
        out = torch.empty((N, Hq, L, Ev), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((N, Hq, L), dtype=torch.float32, device=q.device)
    if tuple(out.shape) != (N, Hq, L, Ev) or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out has the wrong shape/dtype")
    if tuple(lse.shape) != (N, Hq, L) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse has the wrong shape/dtype")
    _same_device(q, k=k, v=v, out=out, lse=lse, sink=sink, bias=bias, mask_bits=mask_bits, kv_start=kv_start,
                 kv_end=kv_end)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        lib = load_library()
        common = (_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), N, Hq, H, L, S, E, Ev, float(scale), MODES[mode],
                  _ptr(sink))
        tail = (_ptr(bias), DTYPES[q.dtype], ctypes.c_void_p(stream.cuda_stream))
        padded = mask_bits is not None or kv_start is not None or kv_end is not None
        if padded:
            if bias is not None or mask_kind == "streaming":
                raise ValueError("mask_bits / kv_start / kv_end combine with none, causal or window masks only, "
                                 "without a bias")
            for name, t, shape in (("mask_bits", mask_bits, (L, (S + 31) // 32)), ("kv_start", kv_start, (N,)),
                                   ("kv_end", kv_end, (N,))):
                if t is not None and (not t.is_cuda or t.dtype != torch.int32 or tuple(t.shape) != shape
                                      or not t.is_contiguous()):
                    raise ValueError(f"{name} must be a contiguous CUDA int32 tensor of shape {shape}")
            st = lib.attn_fwd_padded(*common, MASKS[mask_kind], int(window), _ptr(mask_bits), _ptr(kv_start),
                                     _ptr(kv_end), *tail[1:])
        elif mask_kind == "streaming":
            st = lib.attn_fwd_streaming(*common, int(window), int(keep_first), *tail)
        else:
            st = lib.attn_fwd(*common, MASKS[mask_kind], int(window), *tail)
    _check(st)
    return out, lse


def attn_decode_indexed_raw(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, idx_ptr, n_sel, N, Hq, H, L, S, E, Ev, scale,
                            sink_ptr, mask_kind, window, bias_ptr, stream_ptr) -> int:
    """The index-set decode entry point with integer pointers; returns the status code."""
    lib = load_library()
    c = lambda p: None if p is None else ctypes.c_void_p(int(p))  # noqa: E731
    return lib.attn_decode_indexed(c(q_ptr), c(k_ptr), c(v_ptr), c(out_ptr), c(lse_ptr), c(idx_ptr), int(n_sel),
                                   int(N), int(Hq), int(H), int(L), int(S), int(E), int(Ev), float(scale),
                                   c(sink_ptr), int(mask_kind), int(window), c(bias_ptr), c(stream_ptr))


def attn_decode_indexed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, key_idx: torch.Tensor, *, scale: float,
                        sink: torch.Tensor | None = None, mask_kind: str = "none", window: int = 0,
                        bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        lse: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """Exact decode attention over listed keys.  Returns (out, lse).

    q (N, Hq, L, E), k (N, H, S, E), v (N, H, S, Ev): contiguous bfloat16 CUDA
    tensors with (Hq/H)*L <= 16.  key_idx (N, H, n_sel) int32 CUDA tensor of key
    positions; entries outside [0, S) select nothing.  sink, bias, mask_kind
    ("none", "causal", "window") and window as in attn_fwd.
    """
    _check_kinds("dot", mask_kind, masks=MASKS)
    for name, t in (("q", q), ("k", k), ("v", v), ("key_idx", key_idx)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4 or key_idx.dim() != 3:
        raise ValueError("q, k, v must be 4-D and key_idx 3-D")
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must be bfloat16")
    if key_idx.dtype != torch.int32:
        raise ValueError("key_idx must be int32")
    N, Hq, L, E = q.shape
    _, H, S, _ = k.shape
    Ev = v.shape[3]
    if tuple(key_idx.shape[:2]) != (N, H):
        raise ValueError("key_idx must be (N, H, n_sel)")
    if sink is not None and (sink.dtype != torch.float32 or sink.numel() != Hq or not sink.is_cuda
                             or not sink.is_contiguous()):
        raise ValueError("sink must be a contiguous CUDA float32 tensor of Hq values")
    if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (L, S) or not bias.is_cuda
                             or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous CUDA float32 (L, S) tensor")
    if out is None:
        out = torch.empty((N, Hq, L, Ev), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((N, Hq, L), dtype=torch.float32, device=q.device)
    if tuple(out.shape) != (N, Hq, L, Ev) or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out has the wrong shape/dtype")
    if tuple(lse.shape) != (N, Hq, L) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse has the wrong shape/dtype")
    _same_device(q, k=k, v=v, key_idx=key_idx, out=out, lse=lse, sink=sink, bias=bias)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = load_library().attn_decode_indexed(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(key_idx), key_idx.shape[2], N, Hq, H, L, S, E, Ev,
            float(scale), _ptr(sink), MASKS[mask_kind], int(window), _ptr(bias), ctypes.c_void_p(stream.cuda_stream))
    _check(st)
    return out, lse


def attn_decode_fwd_noalloc_raw(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, N, Hq, H, L, S, E, Ev, scale, mode,
                                sink_ptr, mask_kind, window, bias_ptr, stream_ptr) -> int:
    """The allocation-free decode entry point with integer pointers; returns the status.

    For callers that may not allocate device memory while running: the
    decode partials live in a fixed scratch array inside the library instead
    of an allocated workspace (see include/attn_b200.h)."""
    lib = load_library()
    c = lambda p: None if p is None else ctypes.c_void_p(int(p))  # noqa: E731
    return lib.attn_decode_fwd_noalloc(c(q_ptr), c(k_ptr), c(v_ptr), c(out_ptr), c(lse_ptr), int(N), int(Hq),
                                       int(H), int(L), int(S), int(E), int(Ev), float(scale), int(mode),
                                       c(sink_ptr), int(mask_kind), int(window), c(bias_ptr), c(stream_ptr))


def exp2_poly_eval(x: torch.Tensor) -> torch.Tensor:
    """The softmax's software 2^x applied on the GPU to a float32 CUDA tensor (verification)."""
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    y = torch.empty_like(x)
    _check(load_library().attn_exp2_poly_eval(_ptr(x), _ptr(y), x.numel(),
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))
    return y


def decode_noalloc_scratch_bytes() -> int:
    return int(load_library().attn_decode_noalloc_scratch_bytes())


def inject_wait_timeout(limit_cycles: int, stream: torch.cuda.Stream | None = None) -> int:
    """Failure-path check: a kernel whose one bounded wait runs out (returns the launch status)."""
    s = stream or torch.cuda.current_stream()
    return load_library().attn_test_wait_timeout(int(limit_cycles), ctypes.c_void_p(s.cuda_stream))


def inject_workspace_failures(count: int) -> int:
    """Failure-path check: the next `count` workspace allocations fail (returns the status)."""
    return load_library().attn_test_fail_workspace_allocs(int(count))


def device_status(stream: torch.cuda.Stream | None = None) -> int:
    """Synchronises the stream and returns (and clears) the kernels' fault status."""
    s = stream or torch.cuda.current_stream()
    return load_library().attn_device_status(ctypes.c_void_p(s.cuda_stream))


def release_workspace():
    load_library().attn_release_workspace()


def version() -> int:
    return load_library().attn_version()
