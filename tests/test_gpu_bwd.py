"""Backward pass (gtr_gla_bwd) vs the fp64 oracle's backward (GPU only).

The oracle differentiates the token recurrence position by position
(``oracle.gla_backward``, pinned by tests/test_oracle_bwd.py); both sides read the same
fp16 inputs and upstream gradients.  Cases: every direction on the 1.6K grid with an
initial state and a final-state gradient, ragged grids (a partial last chunk), no
state arguments, dk = 128 (two key halves, grad_v accumulated), strongly forgetting
channels (the per-pair exponential path), gates of exactly 0 and exactly 1, grids
shorter than a chunk, an empty grid, and sampled heads of the 16.4K workload at full
length.

Tolerance: the kernels compute in fp32 from exact fp16 inputs; each gradient element is
a sum of at most a few hundred products per chunk plus chunk-level state scans of at
most a few hundred steps, each step with relative rounding of about 2^-22 (fp32 plus
the exponential's couple of ulp), so the error stays below 2e-4 of the tensor's
largest magnitude; that bound is asserted (and no element may be non-finite).  grad_g
sums q*dq - k*dk over the later positions, so its bound scales with the larger of its
own magnitude and those terms' (with every gate 0 the sum cancels to zero exactly in
fp64 and to rounding in fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import make_inputs, make_upstream

pytestmark = pytest.mark.gpu
REL = 2e-4


def run_both(B, heads, H, W, dk, direction, seed, init_std=0.1, with_dsf=True, heads_sel=None,
             z_mean_per_head=None, want_init_grad=True, z_override=None):
    inp = make_inputs(B, heads, H, W, dk, 64, seed, init_std=init_std, z_mean_per_head=z_mean_per_head,
                      z_override=z_override)
    d_out, dsf = make_upstream(B, heads, H, W, dk, 64, seed, with_dsf=with_dsf)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    s0 = None if inp["s0"] is None else inp["s0"].to(dev)
    grads = gla.gtr_gla_bwd(t["q"], t["k"], t["v"], t["g"], d_out.to(dev), H, W, direction, init_state=s0,
                            d_final_state=None if dsf is None else dsf.to(dev),
                            want_init_grad=want_init_grad)
    torch.cuda.synchronize()
    got = [None if x is None else x.cpu().numpy().astype(np.float64) for x in grads]
    f = lambda x: x.float().numpy()  # noqa: E731  exact upcast
    sel = slice(None) if heads_sel is None else heads_sel
    ref = oracle.gla_backward(f(inp["q"][:, :, sel]), f(inp["k"][:, :, sel]), f(inp["v"][:, :, sel]),
                              f(inp["g"][:, :, sel]), f(d_out[:, :, sel]), H, W, direction,
                              None if inp["s0"] is None else inp["s0"][:, sel].numpy(),
                              None if dsf is None else dsf[:, sel].numpy())
    if heads_sel is not None:   # [B, N, heads, d] gradients, then [B, heads, dk, dv]
        got = [x[:, :, sel] for x in got[:4]] + [None if got[4] is None else got[4][:, sel]]
    # dg sums q*dq - k*dk over the later positions: its rounding scales with those terms
    terms = float(np.max(np.abs(f(inp["q"][:, :, sel]) * ref[0]), initial=0.0)
                  + np.max(np.abs(f(inp["k"][:, :, sel]) * ref[1]), initial=0.0))
    return got, ref + (terms,)


def assert_close(got, ref):
    names = ("grad_q", "grad_k", "grad_v", "grad_g", "grad_init_state")
    for name, x, r in zip(names, got, ref[:5]):
        if x is None:
            continue
        assert np.all(np.isfinite(x)), name
        scale = max(float(np.max(np.abs(r))), ref[5] if name == "grad_g" else 0.0, 1e-30)
        err = float(np.max(np.abs(x - r))) / scale
        assert err <= REL, f"{name}: max|err| / max|ref| = {err:.2e} (> {REL})"


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_every_direction_on_the_1p6k_grid(direction):
    assert_close(*run_both(1, 16, 40, 40, 64, direction, seed=2000 + direction))


@pytest.mark.parametrize("H,W,direction", [(9, 17, 0), (37, 53, 2), (13, 11, 3), (7, 130, 1)])
def test_ragged_grids(H, W, direction):
    assert_close(*run_both(2, 3, H, W, 64, direction, seed=2100 + H))


def test_no_state_arguments():
    got, ref = run_both(1, 4, 20, 20, 64, 0, seed=2200, init_std=None, with_dsf=False)
    assert_close(got, ref)


def test_init_gradient_not_requested():
    got, ref = run_both(1, 4, 20, 20, 64, 1, seed=2250, want_init_grad=False)
    assert got[4] is None
    assert_close(got, ref)


@pytest.mark.parametrize("direction", [2, 3])
def test_dk128_two_key_halves(direction):
    assert_close(*run_both(2, 3, 19, 23, 128, direction, seed=2300 + direction))


def test_strongly_forgetting_channels():
    # z ~ N(-40, 1) on half the heads: chunk decays far below e^-60 (the per-pair path)
    zm = (-40.0, 0.0, -40.0, 4.0)
    assert_close(*run_both(1, 4, 24, 24, 64, 0, seed=2400, z_mean_per_head=zm))


@pytest.mark.parametrize("mode", ["forget_inf", "mixed_inf", "retain"])
def test_degenerate_gates(mode):
    # gates of exactly 0 everywhere (g = -inf in fp16: only each token's own k v
    # survives, and dg is a sum that cancels to zero), gates of exactly 0 scattered
    # among ordinary and extreme ones, and gates of exactly 1 (g = 0)
    def z_of(shape):
        if mode != "mixed_inf":
            return torch.full(shape, -1e38 if mode == "forget_inf" else 60.0)
        gen = torch.Generator().manual_seed(11)
        z = torch.randn(shape, generator=gen) * 40.0
        z[torch.rand(shape, generator=gen) < 0.1] = -1e38
        return z

    for d in (0, 2):
        assert_close(*run_both(1, 4, 20, 20, 64, d, seed=2450, z_override=z_of))


@pytest.mark.parametrize("H,W", [(1, 1), (3, 5), (8, 8)])
def test_grids_within_one_chunk(H, W):
    assert_close(*run_both(1, 2, H, W, 64, 0, seed=2500 + H * W))


def test_empty_grid_passes_the_final_state_gradient():
    dev = torch.device("cuda", 0)
    e16 = torch.empty((1, 0, 2, 64), dtype=torch.float16, device=dev)
    dsf = torch.randn((1, 2, 64, 64), device=dev)
    grads = gla.gtr_gla_bwd(e16, e16, e16, e16, e16, 0, 5, 0, d_final_state=dsf)
    torch.cuda.synchronize()
    assert torch.equal(grads[4], dsf)


def test_full_length_16k_sampled_heads():
    # the 16.4K workload's shape (B1, 16 heads, 128 x 128) at full length; the oracle
    # checks two of the sixteen independent sequences
    got, ref = run_both(1, 16, 128, 128, 64, 3, seed=2600, heads_sel=[0, 11])
    assert_close(got, ref)


def test_repeatable_bit_for_bit():
    a, _ = run_both(1, 4, 24, 24, 64, 2, seed=2700)
    b, _ = run_both(1, 4, 24, 24, 64, 2, seed=2700)
    for x, y in zip(a[:4], b[:4]):
        assert np.array_equal(x, y)
