"""Float64 CPU oracle for the KDA gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY: the independent checker for the GPU library. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this package.
It shares no code with ``gated_delta_rule_144_b200`` and never imports it.

``kda_oracle.cpp`` holds the arithmetic (the per-token recurrence of the GLM-5.3-Flash model
card's Kimi Delta Attention snippet, with packed-document resets as in the NeMo glm5_next
``_torch_recurrent_kda`` docstring). ``brute.py`` is a second, loop-free evaluation used only to
pin the first one on tiny inputs. ``out_norm.py`` is the gated per-head RMSNorm of the output and
``backward.py`` the gradients of the recurrence (the training direction) and ``short_conv.py`` the
short causal convolution of the inputs (with optional SiLU and per-head L2 norm), all float64
NumPy.

Every function here is pinned (tests/test_oracle_pins.py, test_oracle_backward.py,
test_oracle_out_norm.py, test_oracle_short_conv.py); none is "parity unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "kda_oracle.cpp"


def _lib_path(mutant: int = 0) -> Path:
    return _HERE / ("liboracle.so" if mutant == 0 else "liboracle_mutant%d.so" % mutant)


def build(force: bool = False, mutant: int = 0) -> Path:
    """Compile ``kda_oracle.cpp`` into ``liboracle.so`` next to it (gcc, OpenMP, -O2).

    -ffp-contract=off keeps every multiply and add a separately rounded float64 operation.
    ``mutant`` > 0 builds a copy with one planted mistake, for tests/test_oracle_mutants.py only.
    """
    lib = _lib_path(mutant)
    if force or not lib.exists() or lib.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = lib.with_suffix(".so.tmp%d" % os.getpid())
        subprocess.check_call(
            ["g++", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c++17",
             "-DKDA_ORACLE_MUTANT=%d" % mutant, str(_SRC), "-o", str(tmp)])
        os.replace(tmp, lib)
    return lib


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes front of one build of ``kda_oracle.cpp``."""

    def __init__(self, mutant: int = 0):
        path = build(mutant=mutant)
        lib = ctypes.CDLL(str(path))
        i32, p = ctypes.c_int, ctypes.c_void_p
        lib.kda_oracle_fwd.argtypes = [i32, i32, i32, i32, i32, p, p, p, p, p, p, p, i32, p, p,
                                       i32]
        lib.kda_oracle_fwd.restype = i32
        lib.kda_oracle_decode.argtypes = [i32, i32, i32, i32, p, p, p, p, p, p, p, p, i32]
        lib.kda_oracle_decode.restype = i32
        lib.kda_oracle_max_threads.argtypes = []
        lib.kda_oracle_max_threads.restype = i32
        self.lib = lib
        self.mutant = mutant

    def max_threads(self) -> int:
        return int(self.lib.kda_oracle_max_threads())

    def kda_fwd(self, q, k, v, log_g, beta, h0=None, cu_seqlens=None, num_threads: int = 0):
        """Float64 prefill.

        q, k, log_g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; h0: [N, H, dk, dv] or
        None; cu_seqlens: int32 [N + 1] or None (then N = B). Values are taken as float32 (the
        values the GPU sees). Returns (o [B, T, H, dv] float64, hT [N, H, dk, dv] float64).
        """
        q, k, v, log_g, beta = (_f32(x) for x in (q, k, v, log_g, beta))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or log_g.shape != q.shape or v.shape[:3] != q.shape[:3] \
                or beta.shape != q.shape[:3]:
            raise ValueError("inconsistent shapes")
        cu = None
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
            N = cu.shape[0] - 1
        else:
            N = B
        h0a = None if h0 is None else _f32(h0)
        if h0a is not None and h0a.shape != (N, H, dk, dv):
            raise ValueError("h0 must be [N, H, dk, dv]")
        o = np.zeros((B, T, H, dv), dtype=np.float64)
        hT = np.zeros((N, H, dk, dv), dtype=np.float64)
        rc = self.lib.kda_oracle_fwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(log_g),
                                     _ptr(beta), _ptr(h0a), _ptr(cu), N, _ptr(o), _ptr(hT),
                                     int(num_threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments (malformed cu_seqlens or shapes)")
        return o, hT

    def kda_decode(self, q, k, v, log_g, beta, S, num_threads: int = 0):
        """Float64 single-token decode for N sequences.

        q, k, log_g: [N, H, dk]; v: [N, H, dv]; beta: [N, H]; S: [N, H, dk, dv].
        Returns (o [N, H, dv] float64, S_new [N, H, dk, dv] float64). S is not modified.
        """
        q, k, v, log_g, beta, S = (_f32(x) for x in (q, k, v, log_g, beta, S))
        N, H, dk = q.shape
        dv = v.shape[-1]
        if S.shape != (N, H, dk, dv):
            raise ValueError("S must be [N, H, dk, dv]")
        o = np.zeros((N, H, dv), dtype=np.float64)
        S_new = np.zeros((N, H, dk, dv), dtype=np.float64)
        rc = self.lib.kda_oracle_decode(N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(log_g),
                                        _ptr(beta), _ptr(S), _ptr(S_new), _ptr(o),
                                        int(num_threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return o, S_new


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(0)
    return _default


def max_threads() -> int:
    return default().max_threads()


def kda_fwd(*args, **kwargs):
    return default().kda_fwd(*args, **kwargs)


def kda_decode(*args, **kwargs):
    return default().kda_decode(*args, **kwargs)
