"""fp64 CPU oracle for the GTR key-decay gated-linear-attention forward pass and its
backward (reverse-mode differentiation of the same recurrence).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` / reference
leg may import this package.  It shares no code with the CUDA path under
``recurrent_vision_backbone_b200/`` and imports nothing from it.

The arithmetic lives in ``gla_oracle.c`` (token-by-token recurrence in fp64,
OpenMP over the independent (batch, head) sequences); this module only builds
that file with gcc and marshals numpy arrays into it.

What it follows: the GTR news article (tokendh.com), section
"线性注意力到底在省什么" (gated linear attention, forget gate on the key side
only, value-side decay fixed to 1) and section "单向扫描的致命缺陷，以及GTR怎么补"
(four scan directions).  Pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_LIB = os.path.join(_HERE, "libgla_oracle.so")
_lock = threading.Lock()
_lib = None

L2R, R2L, T2B, B2T = 0, 1, 2, 3
DIRECTIONS = {"L2R": L2R, "R2L": R2L, "T2B": T2B, "B2T": B2T}


def compile_oracle(src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the C oracle into a shared library (plain gcc, no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", *extra_flags,
           src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    """Build ``libgla_oracle.so`` next to its source if missing or stale."""
    with _lock:
        stale = (not os.path.exists(_LIB)
                 or os.path.getmtime(_LIB) < os.path.getmtime(_SRC))
        if force or stale:
            compile_oracle()
    return _LIB


def load_library(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gla_oracle_fwd_range.restype = ctypes.c_int
    lib.gla_oracle_fwd_range.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 7 + [
        ctypes.c_long, ctypes.c_long, dp, dp, dp]
    lib.gla_oracle_scan_to_token.restype = ctypes.c_long
    lib.gla_oracle_scan_to_token.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int]
    lib.gla_oracle_gate.restype = ctypes.c_int
    lib.gla_oracle_gate.argtypes = [dp, ctypes.c_long, ctypes.c_double, dp]
    lib.gla_oracle_bwd.restype = ctypes.c_int
    lib.gla_oracle_bwd.argtypes = [dp] * 6 + [ctypes.c_int] * 7 + [dp] * 6
    lib.gla_oracle_max_threads.restype = ctypes.c_int
    lib.gla_oracle_set_threads.argtypes = [ctypes.c_int]
    return lib


def _get():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def scan_to_token(p: int, H: int, W: int, direction: int) -> int:
    return int(_get().gla_oracle_scan_to_token(p, H, W, direction))


def max_threads() -> int:
    return int(_get().gla_oracle_max_threads())


def set_threads(n: int) -> None:
    _get().gla_oracle_set_threads(int(n))


def gla_forward(q, k, v, g, H: int, W: int, direction: int, s0=None,
                p_begin: int = 0, p_end: int | None = None, out=None, lib=None):
    """Run the oracle.

    q, k, g: [B, N, heads, dk]; v: [B, N, heads, dv]; s0: [B, heads, dk, dv] or None.
    Processes scan positions [p_begin, p_end) (default: the whole grid).
    Returns (out [B, N, heads, dv] fp64, s_final [B, heads, dk, dv] fp64).
    Rows of ``out`` for tokens outside the range are zero (or keep the values of
    a caller-supplied ``out``).
    """
    lib = lib or _get()
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    if N != H * W:
        raise ValueError(f"N={N} != H*W={H * W}")
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("shape mismatch between q, k, v, g")
    s0a = None if s0 is None else _f64(s0)
    if s0a is not None and s0a.shape != (B, heads, dk, dv):
        raise ValueError("s0 must be [B, heads, dk, dv]")
    o = np.zeros((B, N, heads, dv)) if out is None else out
    if o.dtype != np.float64 or not o.flags["C_CONTIGUOUS"]:
        raise ValueError("out must be contiguous fp64")
    sf = np.zeros((B, heads, dk, dv))
    pe = N if p_end is None else int(p_end)
    rc = lib.gla_oracle_fwd_range(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, H, W,
                                  dk, dv, int(direction), int(p_begin), pe, _ptr(s0a),
                                  _ptr(o), _ptr(sf))
    if rc != 0:
        raise RuntimeError(f"gla_oracle_fwd_range failed with code {rc}")
    return o, sf


def gla_backward(q, k, v, g, dout, H: int, W: int, direction: int, s0=None, dsf=None,
                 lib=None):
    """Gradients of L = sum(dout * o) + sum(dsf * S_final) through the forward above
    (reverse-mode differentiation of the token recurrence, ``gla_oracle_bwd``).

    q, k, g: [B, N, heads, dk]; v, dout: [B, N, heads, dv]; s0, dsf: [B, heads, dk, dv]
    or None (zero).  Returns (dq, dk, dv, dg, ds0) in fp64, ds0 [B, heads, dk, dv].
    """
    lib = lib or _get()
    q, k, v, g, do = _f64(q), _f64(k), _f64(v), _f64(g), _f64(dout)
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    if N != H * W:
        raise ValueError(f"N={N} != H*W={H * W}")
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3] or do.shape != v.shape:
        raise ValueError("shape mismatch between q, k, v, g, dout")
    s0a = None if s0 is None else _f64(s0)
    dsa = None if dsf is None else _f64(dsf)
    for x in (s0a, dsa):
        if x is not None and x.shape != (B, heads, dk, dv):
            raise ValueError("s0 and dsf must be [B, heads, dk, dv]")
    dq, dkk, dg = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    dvv = np.zeros_like(v)
    ds0 = np.zeros((B, heads, dk, dv))
    rc = lib.gla_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(do), _ptr(dsa), B, heads, H, W,
                            dk, dv, int(direction), _ptr(s0a), _ptr(dq), _ptr(dkk), _ptr(dvv),
                            _ptr(dg), _ptr(ds0))
    if rc != 0:
        raise RuntimeError(f"gla_oracle_bwd failed with code {rc}")
    return dq, dkk, dvv, dg, ds0


def gate(z, tau: float, lib=None) -> np.ndarray:
    """Log-decay of the key-side forget gate from its pre-activation:
    g = log(sigmoid(z)) / tau, in fp64, elementwise (any shape)."""
    lib = lib or _get()
    za = _f64(z)
    g = np.empty_like(za)
    rc = lib.gla_oracle_gate(_ptr(za), za.size, float(tau), _ptr(g))
    if rc != 0:
        raise RuntimeError(f"gla_oracle_gate failed with code {rc}")
    return g


def gla_forward_z(q, k, v, z, tau: float, H: int, W: int, direction: int, s0=None):
    """The forward pass with the gate given by its pre-activation z (fp64 gate, then
    the same recurrence as gla_forward)."""
    return gla_forward(q, k, v, gate(z, tau), H, W, direction, s0)


# ------------------------------------------------------------------ Spatial SwiGLU
# The gated value branch of GTR's Spatial SwiGLU (``swiglu_oracle.c``; the GTR news
# article, section "单向扫描的致命缺陷，以及GTR怎么补").  Its own shared library, built
# the same way.
_SW_SRC = os.path.join(_HERE, "swiglu_oracle.c")
_SW_LIB = os.path.join(_HERE, "libswiglu_oracle.so")
_sw_lib = None


def build_swiglu(force: bool = False) -> str:
    with _lock:
        stale = (not os.path.exists(_SW_LIB)
                 or os.path.getmtime(_SW_LIB) < os.path.getmtime(_SW_SRC))
        if force or stale:
            compile_oracle(_SW_SRC, _SW_LIB)
    return _SW_LIB


def load_swiglu_library(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.swiglu_oracle_gate_conv.restype = ctypes.c_int
    lib.swiglu_oracle_gate_conv.argtypes = [dp, dp, dp, dp] + [ctypes.c_long] * 4 + [dp]
    lib.swiglu_oracle_silu.argtypes = [dp, ctypes.c_long, dp]
    return lib


def _sw():
    global _sw_lib
    if _sw_lib is None:
        _sw_lib = load_swiglu_library(build_swiglu())
    return _sw_lib


def silu(x, lib=None) -> np.ndarray:
    """x * sigmoid(x) in fp64, elementwise."""
    lib = lib or _sw()
    xa = _f64(x)
    y = np.empty_like(xa)
    lib.swiglu_oracle_silu(_ptr(xa), xa.size, _ptr(y))
    return y


def spatial_swiglu_gate(G, U, w, bias=None, lib=None) -> np.ndarray:
    """h = silu(G) * (bias + 3x3 depthwise cross-correlation of U, zero padding).

    G, U: [B, H, W, C]; w: [C, 3, 3]; bias: [C] or None.  Returns h [B, H, W, C] fp64.
    """
    lib = lib or _sw()
    Ga, Ua, wa = _f64(G), _f64(U), _f64(w)
    if Ga.shape != Ua.shape or Ga.ndim != 4:
        raise ValueError("G and U must be [B, H, W, C] of one shape")
    B, H, W, C = Ga.shape
    if wa.shape != (C, 3, 3):
        raise ValueError("w must be [C, 3, 3]")
    ba = None if bias is None else _f64(bias)
    if ba is not None and ba.shape != (C,):
        raise ValueError("bias must be [C]")
    h = np.zeros_like(Ga)
    rc = lib.swiglu_oracle_gate_conv(_ptr(Ga), _ptr(Ua), _ptr(wa), _ptr(ba), B, H, W, C, _ptr(h))
    if rc != 0:
        raise RuntimeError(f"swiglu_oracle_gate_conv failed with code {rc}")
    return h
