"""B200-native Kimi Delta Attention (KDA) gated delta-rule recurrence.

Thin ctypes binding over ``libkda.so`` (C ABI in ``include/kda.h``). This module only marshals
arguments: it checks tensor dtypes and shapes, allocates outputs with PyTorch (PyTorch is used
for device memory and streams only) and passes raw device pointers plus the current CUDA stream
to the library. Every step of the recurrence runs in the library's CUDA kernels; there is no CPU
path. Calling any function without the built library, or with CPU tensors, raises.

Functions mirror the C entry points:
    fwd(q, k, v, log_g, beta, h0=None, cu_seqlens=None, ...)  -> (o, hT)     [kda_fwd]
    decode_step(q, k, v, log_g, beta, S, o=None)               -> o          [kda_decode_step]
    get_device_error(stream=None)                                             [kda_get_device_error]
"""

from __future__ import annotations

import ctypes
from pathlib import Path

import torch

__all__ = ["fwd", "fwd_no_alloc", "out_norm_gated", "short_conv", "decode_step", "decode_tokens",
           "get_device_error",
           "fwd_workspace_size",
           "fwd_workspace_size_min", "fwd_algorithm",
           "KdaError",
           "library_path", "lib", "CHUNK_AUTO", "CHUNK_PER_TOKEN", "CHUNK_64"]

_PKG = Path(__file__).resolve().parent
_LIB_PATH = _PKG / "libkda.so"

CHUNK_AUTO, CHUNK_PER_TOKEN, CHUNK_64 = 0, 1, 64
KDA_F32, KDA_BF16 = 0, 1
STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA",
          4: "KDA_ERR_TIMEOUT", 5: "KDA_ERR_BAD_SEQLENS", 6: "KDA_ERR_RANGE"}


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__("%s: %s%s" % (where, STATUS.get(status, str(status)),
                                       (" (" + detail + ")") if detail else ""))


class FwdDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("num_seqs", ctypes.c_int),
                ("dtype", ctypes.c_int), ("chunk_size", ctypes.c_int)]


class OutNorm(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("eps", ctypes.c_float)]


_lib = None


def library_path() -> Path:
    return _LIB_PATH


def lib():
    """Load libkda.so (once). Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise RuntimeError("libkda.so is missing at %s; build it with "
                           "`python -m gated_delta_rule_144_b200.build`" % _LIB_PATH)
    L = ctypes.CDLL(str(_LIB_PATH))
    p, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.kda_fwd.argtypes = [ctypes.POINTER(FwdDesc), p, p, p, p, p, p, p, p, p, p, sz, p]
    L.kda_fwd.restype = i32
    L.kda_fwd_normed.argtypes = [ctypes.POINTER(FwdDesc), p, p, p, p, p, p, p,
                                 ctypes.POINTER(OutNorm), p, p, p, sz, p]
    L.kda_fwd_normed.restype = i32
    L.kda_out_norm_gated.argtypes = [ctypes.c_longlong, i32, i32, p, p, p, ctypes.c_float, p, p]
    L.kda_out_norm_gated.restype = i32
    L.kda_bwd.argtypes = [ctypes.POINTER(FwdDesc)] + [p] * 16 + [ctypes.c_size_t, p]
    L.kda_bwd.restype = i32
    L.kda_bwd_workspace_size.argtypes = [ctypes.POINTER(FwdDesc)]
    L.kda_bwd_workspace_size.restype = ctypes.c_size_t
    L.kda_short_conv.argtypes = [i32, i32, i32, i32, i32, p, p, p, i32, i32, i32, ctypes.c_float,
                                 p, p]
    L.kda_short_conv.restype = i32
    L.kda_fwd_no_alloc.argtypes = [ctypes.POINTER(FwdDesc), p, p, p, p, p, p, p, p, p, p]
    L.kda_fwd_no_alloc.restype = i32
    L.kda_fwd_algorithm.argtypes = [ctypes.POINTER(FwdDesc), i32]
    L.kda_fwd_algorithm.restype = i32
    L.kda_fwd_split_segments.argtypes = [ctypes.POINTER(FwdDesc), i32]
    L.kda_fwd_split_segments.restype = i32
    L.kda_fwd_scan_segments.argtypes = [ctypes.POINTER(FwdDesc), i32]
    L.kda_fwd_scan_segments.restype = i32
    L.kda_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdDesc)]
    L.kda_fwd_workspace_size.restype = sz
    L.kda_fwd_workspace_size_min.argtypes = [ctypes.POINTER(FwdDesc)]
    L.kda_fwd_workspace_size_min.restype = sz
    L.kda_decode_step.argtypes = [i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p]
    L.kda_decode_step.restype = i32
    L.kda_decode_tokens.argtypes = [i32, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p]
    L.kda_decode_tokens.restype = i32
    L.kda_get_device_error.argtypes = [p]
    L.kda_get_device_error.restype = i32
    L.kda_status_string.argtypes = [i32]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_last_error.argtypes = []
    L.kda_last_error.restype = ctypes.c_char_p
    L.kda_version.argtypes = []
    L.kda_version.restype = i32
    _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        raise KdaError(status, where, lib().kda_last_error().decode(errors="replace"))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError("q/k/v/beta must be bfloat16 or float32, got %s" % t.dtype)


def _dev(t, name, dtype=None, shape=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device.type != "cuda":
        raise ValueError("%s must be a CUDA tensor (the library has no CPU path)" % name)
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def fwd_algorithm(B, T, H, dk, dv, num_seqs, dtype=torch.bfloat16, chunk_size=0,
                  varlen=False) -> int:
    """Path kda_fwd would take: CHUNK_PER_TOKEN or CHUNK_64 (raises KdaError if rejected)."""
    d = FwdDesc(B, T, H, dk, dv, num_seqs, KDA_BF16 if dtype == torch.bfloat16 else KDA_F32,
                chunk_size)
    r = int(lib().kda_fwd_algorithm(ctypes.byref(d), int(varlen)))
    if r < 0:
        _check(-r, "kda_fwd_algorithm")
    return r


def fwd_split_segments(B, T, H, dk, dv, num_seqs, dtype=torch.bfloat16, chunk_size=0,
                       varlen=False) -> int:
    """Chunk segments the split chunked path runs (two kernel launches each)."""
    d = FwdDesc(B, T, H, dk, dv, num_seqs, KDA_BF16 if dtype == torch.bfloat16 else KDA_F32,
                chunk_size)
    r = int(lib().kda_fwd_split_segments(ctypes.byref(d), int(varlen)))
    if r < 0:
        _check(-r, "kda_fwd_split_segments")
    return r


def fwd_scan_segments(B, T, H, dk, dv, num_seqs, dtype=torch.bfloat16, chunk_size=0,
                      varlen=False) -> int:
    """Segments of kda_fwd's two-level state pass for this shape (>= 3), or 1 for the plain
    state pass (``kda_fwd_scan_segments``; host-only, reads KDA_SCAN_SEGMENTS per call)."""
    d = FwdDesc(B, T, H, dk, dv, num_seqs, KDA_BF16 if dtype == torch.bfloat16 else KDA_F32,
                chunk_size)
    r = int(lib().kda_fwd_scan_segments(ctypes.byref(d), int(varlen)))
    if r < 0:
        _check(-r, "kda_fwd_scan_segments")
    return r


def fwd_workspace_size_min(B, T, H, dk, dv, num_seqs, dtype=torch.bfloat16, chunk_size=0) -> int:
    """Smallest workspace kda_fwd accepts (the fused chunked path's document order)."""
    d = FwdDesc(B, T, H, dk, dv, num_seqs, KDA_BF16 if dtype == torch.bfloat16 else KDA_F32,
                chunk_size)
    return int(lib().kda_fwd_workspace_size_min(ctypes.byref(d)))


def fwd_workspace_size(B, T, H, dk, dv, num_seqs, dtype=torch.bfloat16, chunk_size=0) -> int:
    d = FwdDesc(B, T, H, dk, dv, num_seqs, KDA_BF16 if dtype == torch.bfloat16 else KDA_F32,
                chunk_size)
    return int(lib().kda_fwd_workspace_size(ctypes.byref(d)))


def fwd(q, k, v, log_g, beta, h0=None, cu_seqlens=None, *, chunk_size: int = CHUNK_AUTO,
        output_final_state: bool = True, o=None, hT=None, workspace=None, fused: bool = False,
        out_norm=None, stream=None):
    """Prefill (``kda_fwd``): the recurrence over whole sequences or packed documents.

    q, k, log_g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; q/k/v/beta share one dtype
    (bf16 or fp32), log_g is fp32. h0: [N, H, dk, dv] fp32 or None. cu_seqlens: int32 [N + 1]
    on the device (B must be 1) or None. Returns (o [B, T, H, dv], hT [N, H, dk, dv] fp32 or
    None). Outputs may be passed in preallocated. The workspace (a uint8 device tensor) is
    allocated here when not given: kda_fwd_workspace_size bytes (the split chunked path), or,
    with fused=True, only kda_fwd_workspace_size_min bytes (the fused chunked kernel).
    out_norm = (gate, weight, eps) applies the gated per-head RMSNorm (``kda_fwd_normed``): the
    returned output is y = o / sqrt(mean(o^2) + eps) * weight * sigmoid(gate); gate is shaped and
    typed like o, weight is fp32 [dv].
    """
    lib()
    _dev(q, "q")
    dev = q.device
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dt = q.dtype
    _dtype_code(q)
    _dev(k, "k", dt, (B, T, H, dk), dev)
    _dev(log_g, "log_g", torch.float32, (B, T, H, dk), dev)
    _dev(v, "v", dt, None, dev)
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError("v must be [B, T, H, dv]")
    dv = v.shape[3]
    _dev(beta, "beta", dt, (B, T, H), dev)
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor of N + 1 offsets")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    _dev(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _dev(o, "o", dt, (B, T, H, dv), dev)
    if output_final_state:
        if hT is None:
            hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
        else:
            _dev(hT, "hT", torch.float32, (N, H, dk, dv), dev)
    else:
        hT = None
    desc = FwdDesc(B, T, H, dk, dv, N, _dtype_code(q), chunk_size)
    if workspace is None:
        need = int((lib().kda_fwd_workspace_size_min if fused else lib().kda_fwd_workspace_size)(
            ctypes.byref(desc)))
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    else:   # the library picks the path the given size allows
        _dev(workspace, "workspace", torch.uint8, None, dev)
        need = int(lib().kda_fwd_workspace_size_min(ctypes.byref(desc)))
        if workspace.numel() < need:
            raise ValueError("workspace needs at least %d bytes" % need)
    ws_bytes = 0 if workspace is None else workspace.numel()
    if out_norm is not None:
        gate, weight, eps = out_norm
        _dev(gate, "gate", dt, (B, T, H, dv), dev)
        _dev(weight, "weight", torch.float32, (dv,), dev)
        nrm = OutNorm(gate.data_ptr(), weight.data_ptr(), float(eps))
        with torch.cuda.device(dev):
            st = lib().kda_fwd_normed(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(log_g), _ptr(beta), _ptr(h0), _ptr(cu_seqlens),
                                      ctypes.byref(nrm), _ptr(o), _ptr(hT), _ptr(workspace),
                                      ws_bytes, _stream(stream, dev))
        _check(st, "kda_fwd_normed")
        return o, hT
    with torch.cuda.device(dev):
        st = lib().kda_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_g),
                           _ptr(beta), _ptr(h0), _ptr(cu_seqlens), _ptr(o), _ptr(hT),
                           _ptr(workspace), ws_bytes, _stream(stream, dev))
    _check(st, "kda_fwd")
    return o, hT


def bwd_workspace_size(B, T, H, dk, dv, num_seqs, dtype=torch.bfloat16) -> int:
    d = FwdDesc(B, T, H, dk, dv, num_seqs, KDA_BF16 if dtype == torch.bfloat16 else KDA_F32, 0)
    return int(lib().kda_bwd_workspace_size(ctypes.byref(d)))


def bwd(q, k, v, log_g, beta, do, h0=None, dhT=None, cu_seqlens=None, *, workspace=None,
        stream=None):
    """Gradients of the recurrence (``kda_bwd``) for upstream gradients do (of o) and dhT (of
    the final states, or None): returns (dq, dk, dv, dlog_g, dbeta, dh0), all fp32, shaped like
    (q, k, v, log_g, beta, h0 [N, H, dk, dv]). Forward arguments as for ``fwd``; dk = dv = 128.
    dq, dk, dlog_g and dbeta are sums over value-column slices added atomically, so their last
    bits may differ between runs; dv and dh0 are reproducible."""
    lib()
    _dev(q, "q")
    dev = q.device
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dt = q.dtype
    _dtype_code(q)
    _dev(k, "k", dt, (B, T, H, dk), dev)
    _dev(log_g, "log_g", torch.float32, (B, T, H, dk), dev)
    _dev(v, "v", dt, None, dev)
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError("v must be [B, T, H, dv]")
    dv = v.shape[3]
    _dev(beta, "beta", dt, (B, T, H), dev)
    _dev(do, "do", dt, (B, T, H, dv), dev)
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor of N + 1 offsets")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    _dev(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    _dev(dhT, "dhT", torch.float32, (N, H, dk, dv), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = (torch.empty((B, T, H, dk), **f32), torch.empty((B, T, H, dk), **f32),
             torch.empty((B, T, H, dv), **f32), torch.empty((B, T, H, dk), **f32),
             torch.empty((B, T, H), **f32), torch.empty((N, H, dk, dv), **f32))
    desc = FwdDesc(B, T, H, dk, dv, N, _dtype_code(q), 0)
    need = int(lib().kda_bwd_workspace_size(ctypes.byref(desc)))
    if workspace is None:
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    else:
        _dev(workspace, "workspace", torch.uint8, None, dev)
        if workspace.numel() < need:
            raise ValueError("workspace needs at least %d bytes" % need)
    ws_bytes = 0 if workspace is None else workspace.numel()
    with torch.cuda.device(dev):
        st = lib().kda_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_g),
                           _ptr(beta), _ptr(h0), _ptr(cu_seqlens), _ptr(do), _ptr(dhT),
                           *[_ptr(g) for g in grads], _ptr(workspace), ws_bytes,
                           _stream(stream, dev))
    _check(st, "kda_bwd")
    return grads


def out_norm_gated(x, gate, weight, eps: float, *, y=None, stream=None):
    """The gated per-head RMSNorm alone (``kda_out_norm_gated``) over the last axis of x:
    y = x / sqrt(mean(x^2) + eps) * weight * sigmoid(gate). y may be x (in place)."""
    lib()
    _dev(x, "x")
    dev = x.device
    dv = x.shape[-1]
    _dev(gate, "gate", x.dtype, tuple(x.shape), dev)
    _dev(weight, "weight", torch.float32, (dv,), dev)
    if y is None:
        y = torch.empty_like(x)
    else:
        _dev(y, "y", x.dtype, tuple(x.shape), dev)
    with torch.cuda.device(dev):
        st = lib().kda_out_norm_gated(x.numel() // dv, dv, _dtype_code(x), _ptr(x), _ptr(gate),
                                      _ptr(weight), float(eps), _ptr(y), _stream(stream, dev))
    _check(st, "kda_out_norm_gated")
    return y


def _prefill_shapes(q, k, v, log_g, beta, cu_seqlens):
    """(B, T, H, dk, dv, N) of a prefill call; raises ValueError on inconsistent shapes."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    if tuple(k.shape) != (B, T, H, dk) or tuple(log_g.shape) != (B, T, H, dk):
        raise ValueError("k and log_g must be shaped like q, [B, T, H, dk]")
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError("v must be [B, T, H, dv]")
    if tuple(beta.shape) != (B, T, H):
        raise ValueError("beta must be [B, T, H]")
    if cu_seqlens is None:
        return B, T, H, dk, v.shape[3], B
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of N + 1 offsets")
    return B, T, H, dk, v.shape[3], cu_seqlens.numel() - 1


def short_conv(x, weight, cu_seqlens=None, *, activation: str = "none", norm_group: int = 0,
               eps: float = 1e-6, y=None, stream=None):
    """``kda_short_conv``: the short causal convolution of one input (q, k or v) over
    [B, T, C] with a reset at packed-document boundaries, then an optional SiLU
    (activation="silu") and an optional L2 norm of every group of ``norm_group`` channels
    (norm_group = head_dim gives q or k as kda_fwd takes them). weight: fp32 [C, W], W <= 8.
    Returns y shaped and typed like x (y must not be x)."""
    lib()
    _dev(x, "x")
    dev = x.device
    if x.dim() != 3:
        raise ValueError("x must be [B, T, C]")
    B, T, C = x.shape
    _dtype_code(x)
    _dev(weight, "weight", torch.float32, None, dev)
    if weight.dim() != 2 or weight.shape[0] != C:
        raise ValueError("weight must be [C, W]")
    acts = {"none": 0, "silu": 1}
    if activation not in acts:
        raise ValueError("activation must be 'none' or 'silu'")
    N = B
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor of N + 1 offsets")
        N = cu_seqlens.numel() - 1
    if y is None:
        y = torch.empty_like(x)
    else:
        _dev(y, "y", x.dtype, tuple(x.shape), dev)
    with torch.cuda.device(dev):
        st = lib().kda_short_conv(B, T, C, weight.shape[1], _dtype_code(x), _ptr(x), _ptr(weight),
                                  _ptr(cu_seqlens), N, acts[activation], int(norm_group),
                                  float(eps), _ptr(y), _stream(stream, dev))
    _check(st, "kda_short_conv")
    return y


def fwd_no_alloc(q, k, v, log_g, beta, h0, cu_seqlens, o, hT, *, chunk_size: int = CHUNK_AUTO,
                 stream=None):
    """``kda_fwd_no_alloc``: the prefill without a workspace, for callers that cannot allocate.

    Every buffer is the caller's: o [B, T, H, dv] and hT [N, H, dk, dv] (or None) must be passed
    in, and nothing is allocated here or in the library (its scratch is a static device array of
    KDA_NO_ALLOC_MAX_DOCS = 2048 document slots). Calls overlapping on one GPU race on that array.
    Same layouts as ``fwd``; the same results as ``fwd(..., fused=True)``.
    """
    lib()
    # shapes first (no device needed): the library reads v, o and hT with the sizes taken from q
    B, T, H, dk, dv, N = _prefill_shapes(q, k, v, log_g, beta, cu_seqlens)
    for t, name, shape in ((h0, "h0", (N, H, dk, dv)), (o, "o", (B, T, H, dv)),
                           (hT, "hT", (N, H, dk, dv))):
        if t is not None and tuple(t.shape) != shape:
            raise ValueError("%s must have shape %s, got %s" % (name, shape, tuple(t.shape)))
    if o is None:
        raise ValueError("o must be passed in (this entry point allocates nothing)")
    _dev(q, "q")
    dev = q.device
    dt = q.dtype
    _dtype_code(q)
    _dev(k, "k", dt, None, dev)
    _dev(log_g, "log_g", torch.float32, None, dev)
    _dev(v, "v", dt, None, dev)
    _dev(beta, "beta", dt, None, dev)
    _dev(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
    _dev(h0, "h0", torch.float32, None, dev)
    _dev(o, "o", dt, None, dev)
    _dev(hT, "hT", torch.float32, None, dev)
    desc = FwdDesc(B, T, H, dk, dv, N, _dtype_code(q), chunk_size)
    with torch.cuda.device(dev):
        st = lib().kda_fwd_no_alloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_g),
                                    _ptr(beta), _ptr(h0), _ptr(cu_seqlens), _ptr(o), _ptr(hT),
                                    _stream(stream, dev))
    _check(st, "kda_fwd_no_alloc")
    return o, hT


def decode_step(q, k, v, log_g, beta, S, *, o=None, stream=None):
    """One decode token for N sequences (``kda_decode_step``); S is updated in place.

    q, k, log_g: [N, H, dk]; v: [N, H, dv]; beta: [N, H]; S: [N, H, dk, dv] fp32.
    Returns o [N, H, dv] in the dtype of q.
    """
    lib()
    _dev(q, "q")
    dev = q.device
    if q.dim() != 3:
        raise ValueError("q must be [N, H, dk]")
    N, H, dk = q.shape
    dt = q.dtype
    _dtype_code(q)
    _dev(k, "k", dt, (N, H, dk), dev)
    _dev(log_g, "log_g", torch.float32, (N, H, dk), dev)
    _dev(v, "v", dt, None, dev)
    if v.dim() != 3 or tuple(v.shape[:2]) != (N, H):
        raise ValueError("v must be [N, H, dv]")
    dv = v.shape[2]
    _dev(beta, "beta", dt, (N, H), dev)
    _dev(S, "S", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=dt, device=dev)
    else:
        _dev(o, "o", dt, (N, H, dv), dev)
    with torch.cuda.device(dev):
        st = lib().kda_decode_step(N, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(log_g), _ptr(beta), _ptr(S), _ptr(o),
                                   _stream(stream, dev))
    _check(st, "kda_decode_step")
    return o


def decode_tokens(q, k, v, log_g, beta, S, *, o=None, stream=None):
    """T tokens for each of N sequences from their decode state (``kda_decode_tokens``); S is
    updated in place to the state after the last token.

    q, k, log_g: [N, T, H, dk]; v: [N, T, H, dv]; beta: [N, T, H]; S: [N, H, dk, dv] fp32.
    Returns o [N, T, H, dv] in the dtype of q.
    """
    lib()
    _dev(q, "q")
    dev = q.device
    if q.dim() != 4:
        raise ValueError("q must be [N, T, H, dk]")
    N, T, H, dk = q.shape
    dt = q.dtype
    _dtype_code(q)
    _dev(k, "k", dt, (N, T, H, dk), dev)
    _dev(log_g, "log_g", torch.float32, (N, T, H, dk), dev)
    _dev(v, "v", dt, None, dev)
    if v.dim() != 4 or tuple(v.shape[:3]) != (N, T, H):
        raise ValueError("v must be [N, T, H, dv]")
    dv = v.shape[3]
    _dev(beta, "beta", dt, (N, T, H), dev)
    _dev(S, "S", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((N, T, H, dv), dtype=dt, device=dev)
    else:
        _dev(o, "o", dt, (N, T, H, dv), dev)
    with torch.cuda.device(dev):
        st = lib().kda_decode_tokens(N, H, T, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(log_g), _ptr(beta), _ptr(S), _ptr(o),
                                     _stream(stream, dev))
    _check(st, "kda_decode_tokens")
    return o


def get_device_error(stream=None, device=None) -> int:
    """Synchronise and return (then clear) the library's sticky device error code (0 = none)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(lib().kda_get_device_error(_stream(stream, dev)))
