"""Shared helpers for the GPU tests: run the CUDA path and the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from recurrent_vision_backbone_b200 import gla

# Parity bar for floating point: relative to the rms of the fp64 reference,
# over the whole tensor (outputs and final state checked separately).
MAX_REL = 1e-2
MEAN_REL = 1e-3


def run_gpu(inp, H, W, direction, final_state=True, stream=None):
    dev = torch.device("cuda", 0)
    q, k, v, g = (inp[n].to(dev).contiguous() for n in ("q", "k", "v", "g"))
    s0 = None if inp.get("s0") is None else inp["s0"].to(dev).contiguous()
    out, sf = gla.gtr_gla_fwd(q, k, v, g, H, W, direction, init_state=s0,
                              final_state=True if final_state else None, stream=stream)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    return out.float().cpu().numpy(), (None if sf is None else sf.cpu().numpy())


def run_oracle(inp, H, W, direction):
    f = lambda t: t.float().numpy()  # noqa: E731  exact fp16 -> fp32 -> fp64 upcast
    s0 = None if inp.get("s0") is None else inp["s0"].numpy()
    return oracle.gla_forward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["g"]), H, W,
                              direction, s0)


def err_ratios(got, ref):
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0, 0.0, rms
    d = np.abs(got - ref)
    rms = max(rms, 1e-30)
    return float(d.max() / rms), float(d.mean() / rms), rms


def assert_parity(got, ref, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    mx, mn, rms = err_ratios(got, ref)
    assert mx <= MAX_REL and mn <= MEAN_REL, (
        f"{what}: max|err|/rms={mx:.3e} (<= {MAX_REL}), mean|err|/rms={mn:.3e} (<= {MEAN_REL}),"
        f" rms={rms:.3e}")
    return mx, mn
