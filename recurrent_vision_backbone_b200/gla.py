"""Python binding of the C ABI in include/gtr_gla.h, gtr_gla_bwd.h and gtr_swiglu.h
(argument marshalling only).

Every step of the token mixer runs in the CUDA library ``libgtr_gla.so``; this
module only checks tensor metadata, passes raw device pointers and the CUDA
stream through ``ctypes``, and turns status codes into exceptions.  There is no
CPU or PyTorch fallback: if the library is missing or no GPU is present the
calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgtr_gla.so")

GTR_OK, GTR_ERR_INVALID_ARG, GTR_ERR_UNSUPPORTED, GTR_ERR_CUDA, GTR_ERR_TIMEOUT, GTR_ERR_RANGE = range(6)
L2R, R2L, T2B, B2T = 0, 1, 2, 3
STATIC_WS_BYTES = 4 << 20   # GTR_STATIC_WS_BYTES

EXPORTED_SYMBOLS = ("gtr_gla_fwd", "gtr_gla_fwd_z", "gtr_gla_fwd_stack", "gtr_gla_init", "gtr_gla_workspace_bytes", "gtr_gla_fwd_ws",
                    "gtr_gla_fwd_static", "gtr_gla_device_status", "gtr_status_str", "gtr_gla_plan", "gtr_gla_version",
                    "gtr_gla_last_error", "gtr_gla_selftest_timeout", "gtr_spatial_swiglu_gate",
                    "gtr_gla_bwd", "gtr_gla_bwd_workspace_bytes")

_lock = threading.Lock()
_lib = None


class Layer(ctypes.Structure):
    """gtr_gla_layer_t: one layer call of a stack (device pointers and a direction)."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("init_state", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("final_state", ctypes.c_void_p), ("direction", ctypes.c_int)]


class GTRError(RuntimeError):
    def __init__(self, status: int, where: str):
        detail = ""
        if status == GTR_ERR_CUDA and _lib is not None:
            detail = f" [{_lib.gtr_gla_last_error().decode()}]"
        super().__init__(f"{where}: {status_str(status)} (status {status}){detail}")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m recurrent_vision_backbone_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i = ctypes.c_void_p, ctypes.c_int
        lib.gtr_gla_fwd.restype = i
        lib.gtr_gla_fwd.argtypes = [vp, vp, vp, vp] + [i] * 8 + [vp, vp, vp, vp]
        lib.gtr_gla_fwd_z.restype = i
        lib.gtr_gla_fwd_z.argtypes = [vp, vp, vp, vp, ctypes.c_float] + [i] * 8 + [vp, vp, vp, vp]
        lib.gtr_spatial_swiglu_gate.restype = i
        lib.gtr_spatial_swiglu_gate.argtypes = [vp, vp, vp, vp] + [i] * 4 + [vp, vp]
        lib.gtr_gla_fwd_stack.restype = i
        lib.gtr_gla_fwd_stack.argtypes = [ctypes.POINTER(Layer)] + [i] * 8 + [vp]
        lib.gtr_gla_fwd_static.restype = i
        lib.gtr_gla_fwd_static.argtypes = [vp, vp, vp, vp] + [i] * 8 + [vp, vp, vp, vp]
        lib.gtr_gla_workspace_bytes.restype = ctypes.c_size_t
        lib.gtr_gla_workspace_bytes.argtypes = [i] * 7
        lib.gtr_gla_fwd_ws.restype = i
        lib.gtr_gla_fwd_ws.argtypes = ([vp, vp, vp, vp] + [i] * 8 + [vp, vp, vp]
                                       + [vp, ctypes.c_size_t, vp])
        lib.gtr_gla_bwd.restype = i
        lib.gtr_gla_bwd.argtypes = [vp] * 7 + [i] * 8 + [vp] * 6 + [ctypes.c_size_t, vp]
        lib.gtr_gla_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.gtr_gla_bwd_workspace_bytes.argtypes = [i] * 7
        lib.gtr_gla_device_status.restype = i
        lib.gtr_gla_device_status.argtypes = [vp]
        lib.gtr_gla_init.restype = i
        lib.gtr_gla_init.argtypes = [vp]
        lib.gtr_gla_selftest_timeout.restype = i
        lib.gtr_gla_selftest_timeout.argtypes = [ctypes.c_uint, vp]
        lib.gtr_status_str.restype = ctypes.c_char_p
        lib.gtr_status_str.argtypes = [i]
        lib.gtr_gla_plan.restype = i
        ip = ctypes.POINTER(ctypes.c_int)
        lib.gtr_gla_plan.argtypes = [i] * 6 + [ip, ip, ip]
        lib.gtr_gla_version.restype = ctypes.c_char_p
        lib.gtr_gla_last_error.restype = ctypes.c_char_p
        _lib = lib
        return lib


def status_str(status: int) -> str:
    try:
        return load().gtr_status_str(int(status)).decode()
    except Exception:  # library not loadable: plain text
        return {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
                4: "device-side wait timed out",
                5: "an fp16 operand or output left the fp16 range"}.get(int(status), "unknown status")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _prepare(q, k, v, g, Hgrid, Wgrid, init_state, out, final_state):
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("g", g), ("v", v)):
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA float16 tensor")
    # the library launches on the current device: every tensor must live there
    cur = torch.cuda.current_device()
    for name, t in (("q", q), ("k", k), ("g", g), ("v", v), ("init_state", init_state),
                    ("out", out), ("final_state", None if final_state is True else final_state)):
        if t is not None and t.device.index != cur:
            raise ValueError(f"{name} is on {t.device}, but the current CUDA device is cuda:{cur}")
    if k.shape != q.shape or g.shape != q.shape or tuple(v.shape[:3]) != (B, N, heads):
        raise ValueError("q, k, g must be [B,N,heads,dk] and v [B,N,heads,dv]")
    if N != Hgrid * Wgrid:
        raise ValueError(f"N={N} does not match the grid {Hgrid}x{Wgrid}")
    if out is None:
        out = torch.empty((B, N, heads, dv), dtype=torch.float16, device=q.device)
    if final_state is True:
        final_state = torch.empty((B, heads, dk, dv), dtype=torch.float32, device=q.device)
    for name, t in (("init_state", init_state), ("final_state", final_state)):
        if t is not None and (t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous()
                              or tuple(t.shape) != (B, heads, dk, dv)):
            raise ValueError(f"{name} must be a contiguous CUDA float32 [B,heads,dk,dv] tensor")
    return (B, heads, dk, dv), out, final_state


def gtr_gla_fwd(q, k, v, g, Hgrid: int, Wgrid: int, direction: int, init_state=None,
                out=None, final_state=None, chunk: int = 64, stream=None):
    """One token-mixer call on device tensors.

    q, k, g: fp16 [B, N, heads, dk]; v: fp16 [B, N, heads, dv] (CUDA, contiguous).
    init_state: fp32 [B, heads, dk, dv] or None.  final_state: an fp32 tensor to
    fill, True to allocate one, or None to skip it.  Returns (out, final_state).
    """
    lib = load()
    (B, heads, dk, dv), out, final_state = _prepare(q, k, v, g, Hgrid, Wgrid, init_state, out,
                                                    final_state)
    st = lib.gtr_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, Hgrid, Wgrid, dk, dv,
                         int(direction), int(chunk), _ptr(init_state), _ptr(out),
                         _ptr(final_state), _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_fwd")
    return out, final_state


def gtr_gla_fwd_z(q, k, v, z, tau: float, Hgrid: int, Wgrid: int, direction: int,
                  init_state=None, out=None, final_state=None, chunk: int = 64, stream=None):
    """gtr_gla_fwd with the gate's pre-activation z (fp16, the layout of g) and its
    temperature tau: the kernel forms g = log(sigmoid(z)) / tau in fp32 wherever it reads the gate."""
    (B, heads, dk, dv), out, final_state = _prepare(q, k, v, z, Hgrid, Wgrid, init_state, out,
                                                    final_state)
    st = load().gtr_gla_fwd_z(_ptr(q), _ptr(k), _ptr(v), _ptr(z), ctypes.c_float(tau), B, heads,
                              Hgrid, Wgrid, dk, dv, int(direction), int(chunk), _ptr(init_state),
                              _ptr(out), _ptr(final_state), _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_fwd_z")
    return out, final_state


def gtr_spatial_swiglu_gate(G, U, w, bias=None, out=None, stream=None):
    """Gated value branch of Spatial SwiGLU: silu(G) * (bias + 3x3 depthwise
    cross-correlation of U, zero padding).  G, U: fp16 [B, H, W, C] on the GPU;
    w: fp32 [C, 3, 3]; bias: fp32 [C] or None.  Returns out (fp16, like G)."""
    import torch
    if G.shape != U.shape or G.dim() != 4:
        raise ValueError("G and U must be [B, H, W, C] of one shape")
    B, H, W, C = G.shape
    for name, t in (("G", G), ("U", U)):
        if t.dtype != torch.float16 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous fp16 CUDA tensor")
    if tuple(w.shape) != (C, 3, 3) or w.dtype != torch.float32 or not w.is_contiguous() or w.device != G.device:
        raise ValueError("w must be a contiguous fp32 [C, 3, 3] tensor on G's device")
    if bias is not None and (tuple(bias.shape) != (C,) or bias.dtype != torch.float32 or
                             not bias.is_contiguous() or bias.device != G.device):
        raise ValueError("bias must be a contiguous fp32 [C] tensor on G's device")
    if out is None:
        out = torch.empty_like(G)
    st = load().gtr_spatial_swiglu_gate(_ptr(G), _ptr(U), _ptr(w), _ptr(bias), B, H, W, C, _ptr(out),
                                        _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_spatial_swiglu_gate")
    return out


def gtr_gla_fwd_stack(layers, Hgrid: int, Wgrid: int, chunk: int = 64, stream=None):
    """A stack of layer calls of one shape, in order (see gtr_gla_fwd_stack in the header).

    layers: sequence of dicts with q, k, v, g (fp16 [B,N,heads,d]), direction, and optional
    init_state, out, final_state (final_state=True allocates one).  Returns the list of
    (out, final_state) per layer."""
    arr = (Layer * len(layers))()
    results = []
    shape = None
    for i, L in enumerate(layers):
        sh, out, fs = _prepare(L["q"], L["k"], L["v"], L["g"], Hgrid, Wgrid, L.get("init_state"),
                               L.get("out"), L.get("final_state"))
        if shape is not None and sh != shape:
            raise ValueError("every layer of a stack has the same shape")
        shape = sh
        arr[i] = Layer(L["q"].data_ptr(), L["k"].data_ptr(), L["v"].data_ptr(), L["g"].data_ptr(),
                       None if L.get("init_state") is None else L["init_state"].data_ptr(),
                       out.data_ptr(), None if fs is None else fs.data_ptr(), int(L["direction"]))
        results.append((out, fs))
    B, heads, dk, dv = shape
    st = load().gtr_gla_fwd_stack(arr, len(layers), B, heads, Hgrid, Wgrid, dk, dv, int(chunk),
                                  _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_fwd_stack")
    return results


def gtr_gla_fwd_static(q, k, v, g, Hgrid: int, Wgrid: int, direction: int, init_state=None,
                       out=None, final_state=None, chunk: int = 64, stream=None):
    """gtr_gla_fwd whose workspace is the library's static device scratch (no allocation
    by the library; calls must not overlap in time).  Shapes whose plan needs more than
    STATIC_WS_BYTES raise GTRError(GTR_ERR_UNSUPPORTED)."""
    lib = load()
    (B, heads, dk, dv), out, final_state = _prepare(q, k, v, g, Hgrid, Wgrid, init_state, out,
                                                    final_state)
    st = lib.gtr_gla_fwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, Hgrid, Wgrid, dk,
                                dv, int(direction), int(chunk), _ptr(init_state), _ptr(out),
                                _ptr(final_state), _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_fwd_static" + (
            f" (plan needs more than the {STATIC_WS_BYTES}-byte static scratch)"
            if st == GTR_ERR_UNSUPPORTED and dk == 64 and dv == 64 and chunk == 64 else ""))
    return out, final_state


def workspace_bytes(B: int, heads: int, Hgrid: int, Wgrid: int, dk: int, dv: int,
                    chunk: int = 64) -> int:
    """Workspace gtr_gla_fwd_ws needs for a shape on the current device (0: none)."""
    return int(load().gtr_gla_workspace_bytes(B, heads, Hgrid, Wgrid, dk, dv, chunk))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled device buffer usable as a workspace (at least one byte)."""
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def gtr_gla_fwd_ws(q, k, v, g, Hgrid: int, Wgrid: int, direction: int, workspace,
                   init_state=None, out=None, final_state=None, chunk: int = 64, stream=None):
    """gtr_gla_fwd with a caller-owned workspace (a CUDA uint8 tensor or None)."""
    lib = load()
    (B, heads, dk, dv), out, final_state = _prepare(q, k, v, g, Hgrid, Wgrid, init_state, out,
                                                    final_state)
    if workspace is not None and (not workspace.is_cuda or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.gtr_gla_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, Hgrid, Wgrid, dk, dv,
                            int(direction), int(chunk), _ptr(init_state), _ptr(out),
                            _ptr(final_state), _ptr(workspace), nbytes, _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_fwd_ws")
    return out, final_state


def bwd_workspace_bytes(B: int, heads: int, Hgrid: int, Wgrid: int, dk: int, dv: int,
                        chunk: int = 64) -> int:
    """Workspace gtr_gla_bwd needs for a shape (0: none, or a rejected shape)."""
    return int(load().gtr_gla_bwd_workspace_bytes(B, heads, Hgrid, Wgrid, dk, dv, chunk))


def gtr_gla_bwd(q, k, v, g, d_out, Hgrid: int, Wgrid: int, direction: int, init_state=None,
                d_final_state=None, workspace=None, grads=None, want_init_grad: bool = True,
                chunk: int = 64, stream=None):
    """Backward pass of one token-mixer call on device tensors.

    q, k, g, v, init_state, Hgrid, Wgrid, direction: as given to the forward call;
    d_out: fp16 [B, N, heads, dv] = dL/do; d_final_state: fp32 [B, heads, dk, dv] or None.
    workspace: a CUDA uint8 tensor of at least bwd_workspace_bytes(...) bytes, or None
    to allocate one.  grads: a tuple (grad_q, grad_k, grad_v, grad_g, grad_init_state) of
    fp32 tensors to fill, or None to allocate them.  Returns that tuple (grad_init_state
    None unless want_init_grad).
    """
    lib = load()
    (B, heads, dk, dv), _, _ = _prepare(q, k, v, g, Hgrid, Wgrid, init_state, d_out, None)
    N = q.shape[1]
    if d_out.dtype != torch.float16 or not d_out.is_contiguous() or tuple(d_out.shape) != tuple(v.shape):
        raise ValueError("d_out must be a contiguous CUDA float16 tensor shaped like v")
    if d_final_state is not None and (d_final_state.dtype != torch.float32 or not d_final_state.is_contiguous()
                                      or tuple(d_final_state.shape) != (B, heads, dk, dv)
                                      or d_final_state.device != q.device):
        raise ValueError("d_final_state must be a contiguous float32 [B,heads,dk,dv] tensor on q's device")
    if grads is None:
        f32 = dict(dtype=torch.float32, device=q.device)
        grads = (torch.empty((B, N, heads, dk), **f32), torch.empty((B, N, heads, dk), **f32),
                 torch.empty((B, N, heads, dv), **f32), torch.empty((B, N, heads, dk), **f32),
                 torch.empty((B, heads, dk, dv), **f32) if want_init_grad else None)
    for name, t, shape in zip(("grad_q", "grad_k", "grad_v", "grad_g", "grad_init_state"), grads,
                              ((B, N, heads, dk), (B, N, heads, dk), (B, N, heads, dv), (B, N, heads, dk),
                               (B, heads, dk, dv))):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != shape
                              or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous float32 {list(shape)} tensor on q's device")
    if workspace is None:
        workspace = new_workspace(bwd_workspace_bytes(B, heads, Hgrid, Wgrid, dk, dv, chunk), q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    nbytes = workspace.numel() * workspace.element_size()
    gq, gk, gv, gg, gs = grads
    st = lib.gtr_gla_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(d_out), _ptr(init_state),
                         _ptr(d_final_state), B, heads, Hgrid, Wgrid, dk, dv, int(direction), int(chunk),
                         _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gg), _ptr(gs), _ptr(workspace), nbytes,
                         _stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_bwd")
    return grads


def gtr_gla_fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, g_ptr: int, B: int, heads: int,
                    Hgrid: int, Wgrid: int, dk: int, dv: int, direction: int, chunk: int,
                    init_ptr: int, out_ptr: int, final_ptr: int, stream_handle: int) -> int:
    """Direct pass-through of raw pointers; returns the status code."""
    return load().gtr_gla_fwd(ctypes.c_void_p(q_ptr), ctypes.c_void_p(k_ptr),
                              ctypes.c_void_p(v_ptr), ctypes.c_void_p(g_ptr), B, heads, Hgrid,
                              Wgrid, dk, dv, direction, chunk,
                              ctypes.c_void_p(init_ptr) if init_ptr else None,
                              ctypes.c_void_p(out_ptr),
                              ctypes.c_void_p(final_ptr) if final_ptr else None,
                              ctypes.c_void_p(stream_handle))


def init(stream=None) -> None:
    """Allocate the library's cached workspace of the current device now (stream-ordered),
    e.g. before capturing calls into a CUDA graph."""
    st = load().gtr_gla_init(_stream_handle(stream))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_init")


def device_status(stream=None) -> int:
    """Sync the stream; return (and clear) the device error status."""
    return int(load().gtr_gla_device_status(_stream_handle(stream)))


def selftest_timeout(limit_us: int = 2000, stream=None) -> int:
    """Enqueue the device failure-path self-test (waits that nothing satisfies, bounded
    by limit_us); the next device_status() reports GTR_ERR_TIMEOUT.  Returns the
    launch status."""
    return int(load().gtr_gla_selftest_timeout(int(limit_us), _stream_handle(stream)))


def plan(B: int, heads: int, Hgrid: int, Wgrid: int, dk: int, dv: int):
    """(CTAs per sequence, CTA groups, smem_bytes) the library would launch with."""
    lib = load()
    a, b, c = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = lib.gtr_gla_plan(B, heads, Hgrid, Wgrid, dk, dv, ctypes.byref(a), ctypes.byref(b),
                          ctypes.byref(c))
    if st != GTR_OK:
        raise GTRError(st, "gtr_gla_plan")
    return a.value, b.value, c.value


def version() -> str:
    return load().gtr_gla_version().decode()
