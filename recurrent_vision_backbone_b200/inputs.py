"""Seeded synthetic inputs for the GTR token-mixer forward pass.

This module holds the workload table and the input recipe only: it draws
random tensors and performs none of the token mixer's arithmetic, so that both
the CUDA path's tests/bench and the fp64 oracle can consume the same inputs.

Recipe (one call of one workload):
  * a ``torch.Generator`` seeded per (workload, direction, call) draws, in this
    order and in C order over the full tensors, fp32 standard normals for
    q [B,N,heads,dk], k [B,N,heads,dk], v [B,N,heads,dv], z [B,N,heads,dk] and,
    when the workload has one, the initial state S0 [B,heads,dk,dv];
  * q is scaled by dk**-0.5; z gets a per-head mean shift where the workload
    says so; the forget-gate log-decay is g = logsigmoid(z) / tau with tau = 16
    (the gate parameterisation of the key-side forget gate, GTR news article,
    section "线性注意力到底在省什么"); S0 is scaled by its std (0.1);
  * q, k, v, g are cast to fp16 (round to nearest even); S0 stays fp32.
Both sides read the identical rounded values.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch
import torch.nn.functional as F

L2R, R2L, T2B, B2T = 0, 1, 2, 3
DIR_NAMES = ("L2R", "R2L", "T2B", "B2T")
TAU = 16.0


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int                   # 1-based position in the workload table
    name: str
    B: int
    heads: int
    H: int
    W: int
    dk: int
    dv: int
    directions: tuple            # scan directions exercised by this workload
    calls: int = 1               # layer calls per direction pass (12 for the stacked case)
    init_std: Optional[float] = None   # None: zero initial state
    final_state: bool = False
    z_mean_per_head: Optional[tuple] = None
    fixed_seed: Optional[int] = None   # the first workload fixes its seed

    @property
    def N(self) -> int:
        return self.H * self.W

    @property
    def n_seq(self) -> int:
        return self.B * self.heads

    def tokens(self) -> int:
        """Spatial tokens per layer call (all heads share a token)."""
        return self.B * self.N

    def seed(self, direction: int, call: int = 0) -> int:
        if self.fixed_seed is not None:
            return self.fixed_seed + 10 * direction + call
        return 1000 * self.index + 10 * direction + call

    def call_directions(self) -> Sequence[int]:
        """Directions of the successive calls (cycled when calls > 1)."""
        if self.calls == 1:
            return list(self.directions)
        return [self.directions[c % len(self.directions)] for c in range(self.calls)]


WORKLOADS = {
    w.name: w
    for w in (
        Workload(1, "pr1_b1h4_20x20", 1, 4, 20, 20, 64, 64, (L2R,), fixed_seed=0),
        Workload(2, "gtr640_b1h16_40x40", 1, 16, 40, 40, 64, 64, (L2R, R2L, T2B, B2T),
                 final_state=True),
        Workload(3, "b8h16_48x48_stack12", 8, 16, 48, 48, 64, 64, (L2R, R2L, T2B, B2T),
                 calls=12),
        Workload(4, "hires_b1h16_128x128", 1, 16, 128, 128, 64, 64, (L2R, R2L, T2B, B2T),
                 init_std=0.1, final_state=True),
        Workload(5, "stress_b4h12_37x53_dk128", 4, 12, 37, 53, 128, 64, (T2B, B2T),
                 z_mean_per_head=(4.0,) * 6 + (-4.0,) * 6),
    )
}


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        for w in WORKLOADS.values():
            if w.index == name_or_index:
                return w
        raise KeyError(name_or_index)
    return WORKLOADS[name_or_index]


def make_inputs(B: int, heads: int, H: int, W: int, dk: int, dv: int, seed: int,
                init_std: Optional[float] = None, z_mean_per_head=None,
                device="cpu", z_override=None, with_z=False):
    """Draw one call's inputs following the module recipe.

    Returns dict(q, k, v, g: fp16 tensors [B,N,heads,d]; s0: fp32 [B,heads,dk,dv]
    or None).  ``device`` selects where the generator runs (CPU by default, so
    that CPU and GPU consumers see bit-identical values).
    ``z_override`` (optional callable shape -> fp32 tensor) replaces the gate
    pre-activation draw, for edge cases such as all-retain or all-forget gates.
    ``with_z`` also returns the pre-activation itself (fp16, "z"), for the entry point
    that forms g from it.
    """
    N = H * W
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    kw = dict(generator=gen, device=device, dtype=torch.float32)
    q = torch.randn((B, N, heads, dk), **kw)
    k = torch.randn((B, N, heads, dk), **kw)
    v = torch.randn((B, N, heads, dv), **kw)
    z = torch.randn((B, N, heads, dk), **kw)
    s0 = torch.randn((B, heads, dk, dv), **kw) * float(init_std) if init_std else None
    q = q * (dk ** -0.5)
    if z_mean_per_head is not None:
        mu = torch.tensor(z_mean_per_head, dtype=torch.float32, device=device)
        z = z + mu.view(1, 1, heads, 1)
    if z_override is not None:
        z = z_override((B, N, heads, dk)).to(device=device, dtype=torch.float32)
    g = F.logsigmoid(z) / TAU
    out = dict(q=q.half(), k=k.half(), v=v.half(), g=g.half(), s0=s0)
    if with_z:
        out["z"] = z.half()
    return out


def workload_inputs(w: Workload, direction: int, call: int = 0, device="cpu"):
    return make_inputs(w.B, w.heads, w.H, w.W, w.dk, w.dv, w.seed(direction, call),
                       init_std=w.init_std, z_mean_per_head=w.z_mean_per_head,
                       device=device)


def make_upstream(B: int, heads: int, H: int, W: int, dk: int, dv: int, seed: int,
                  with_dsf: bool = True, device="cpu"):
    """Upstream gradients for the backward pass: d_out = dL/do (fp16 [B,N,heads,dv]) and
    d_final_state = dL/dS_final (fp32 [B,heads,dk,dv] or None), both N(0, 1) -- the scale
    of a squared-L2 loss's gradient on unit-scale features (the pages distil with such a
    loss).  Drawn from their own generator, seeded `seed` + 7, after the forward inputs."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) + 7)
    kw = dict(generator=gen, device=device, dtype=torch.float32)
    d_out = torch.randn((B, H * W, heads, dv), **kw).half()
    dsf = torch.randn((B, heads, dk, dv), **kw) if with_dsf else None
    return d_out, dsf


# ------------------------------------------------------------------ Spatial SwiGLU
# Inputs of the gated value branch (gtr_spatial_swiglu_gate): the gate and up
# projections G, U of a block's tokens and the depthwise kernel.  The pages give no
# block width; the recipe reads the token mixer's 16 heads x 64 channels = 1024 as the
# block width and a hidden width of 2x that, 2048 (the SwiGLU's two projections).
# G, U ~ N(0, 1) cast to fp16; w ~ N(0, 1/9) (a 3x3 kernel's fan-in) and bias ~
# N(0, 0.1^2) in fp32.  The grids are the token mixer's: 40x40 (1.6K tokens) and the
# 768px batch, B8 48x48.
@dataclasses.dataclass(frozen=True)
class SwigluWorkload:
    name: str
    B: int
    H: int
    W: int
    C: int

    @property
    def N(self):
        return self.H * self.W


SWIGLU_WORKLOADS = {w.name: w for w in (
    SwigluWorkload("swiglu_b1_40x40_c2048", 1, 40, 40, 2048),
    SwigluWorkload("swiglu_b8_48x48_c2048", 8, 48, 48, 2048),
)}


def make_swiglu_inputs(B: int, H: int, W: int, C: int, seed: int, bias: bool = True, device="cpu"):
    """Draw G, U (fp16 [B, H, W, C]), w (fp32 [C, 3, 3]) and bias (fp32 [C] or None)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    kw = dict(generator=gen, device=device, dtype=torch.float32)
    G = torch.randn((B, H, W, C), **kw)
    U = torch.randn((B, H, W, C), **kw)
    w = torch.randn((C, 3, 3), **kw) / 3.0
    b = torch.randn((C,), **kw) * 0.1 if bias else None
    return dict(G=G.half(), U=U.half(), w=w, bias=b)
