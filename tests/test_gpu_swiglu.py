"""Spatial SwiGLU gated value branch: gtr_spatial_swiglu_gate vs the fp64 oracle,
element by element (GPU only).

out = silu(G) * (bias + 3x3 depthwise cross-correlation of U, zero padding).  Shapes
cover whole and ragged 16x16 pixel tiles, channel counts that are not a multiple of
the 64-channel tile, one-pixel grids, a batch, no bias, in place over G, the two full
workloads of the recipe, and the argument and range errors.
"""
import numpy as np
import pytest
import torch

import oracle
from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import SWIGLU_WORKLOADS, make_swiglu_inputs
pytestmark = pytest.mark.gpu


def assert_parity(got, ref, what, mag):
    """The bar this op's arithmetic fixes: inputs reach both sides as the same fp16
    values and the kernel sums nine products and the bias in fp32, so the error is
    the final rounding to fp16 — at most half a unit in the last place, 2^-11 |ref|
    for normal results, 6e-8 for fp16 subnormals — plus the fp32 sum's error (below
    1e-6 of |silu(G)| (|bias| + sum |w| |U|), `mag`, the oracle run on magnitudes)
    and the SiLU's (__expf, reciprocal: below 4e-6 relative).  Checked element by
    element (a max|err|/rms bar cannot hold here: with 37.7M outputs the largest
    reach ~100 rms, where half an fp16 ulp is 2e-2 rms)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    bound = (2.0 ** -11 + 4e-6) * np.abs(ref) + 1e-6 * np.abs(mag) + 6e-8
    err = np.abs(got - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} outside half an fp16 ulp; worst at {i}: "
                             f"got {got[i]!r}, ref {ref[i]!r}")
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    assert float(err.mean()) <= 1e-3 * max(rms, 1e-30), what


def _run(inp, in_place=False):
    dev = torch.device("cuda", 0)
    G, U, w = inp["G"].to(dev), inp["U"].to(dev), inp["w"].to(dev)
    bias = None if inp["bias"] is None else inp["bias"].to(dev)
    out = gla.gtr_spatial_swiglu_gate(G, U, w, bias, out=G if in_place else None)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    return out.float().cpu().numpy()


def _oracle(inp):
    """(reference, magnitude of the summed terms) from the fp64 oracle."""
    b = None if inp["bias"] is None else inp["bias"].double().numpy()
    G, U, w = inp["G"].float().numpy(), inp["U"].float().numpy(), inp["w"].double().numpy()
    ref = oracle.spatial_swiglu_gate(G, U, w, b)
    mag = oracle.spatial_swiglu_gate(G, np.abs(U), np.abs(w), None if b is None else np.abs(b))
    return ref, mag


SHAPES = [
    # B, H, W, C, bias
    (1, 16, 16, 64, True),     # one whole tile
    (1, 17, 33, 64, True),     # ragged tiles in both directions
    (2, 9, 7, 128, False),     # a batch, a grid smaller than a tile, no bias
    (1, 1, 1, 64, True),       # one pixel: only the centre tap
    (1, 5, 40, 72, True),      # 72 channels: a partial second channel tile
    (1, 21, 3, 8, True),       # 8 channels
    (3, 12, 19, 200, True),    # 200 channels
]


@pytest.mark.parametrize("B,H,W,C,bias", SHAPES)
def test_shapes_match_oracle(B, H, W, C, bias):
    inp = make_swiglu_inputs(B, H, W, C, seed=H * 131 + W * 7 + C, bias=bias)
    ref, mag = _oracle(inp)
    assert_parity(_run(inp), ref, f"{B}x{H}x{W}x{C}", mag)


def test_in_place_over_gate():
    inp = make_swiglu_inputs(1, 20, 24, 128, seed=5)
    ref, mag = _oracle(inp)
    assert_parity(_run(inp, in_place=True), ref, "in place", mag)


@pytest.mark.parametrize("name", sorted(SWIGLU_WORKLOADS))
def test_workloads_match_oracle(name):
    w = SWIGLU_WORKLOADS[name]
    inp = make_swiglu_inputs(w.B, w.H, w.W, w.C, seed=77)
    ref, mag = _oracle(inp)
    assert_parity(_run(inp), ref, name, mag)


def test_deterministic():
    inp = make_swiglu_inputs(2, 33, 17, 192, seed=9)
    assert np.array_equal(_run(inp), _run(inp))


def test_argument_errors_and_range():
    dev = torch.device("cuda", 0)
    G = torch.zeros((1, 4, 4, 12), dtype=torch.float16, device=dev)
    w = torch.zeros((12, 3, 3), dtype=torch.float32, device=dev)
    with pytest.raises(gla.GTRError) as e:
        gla.gtr_spatial_swiglu_gate(G, G.clone(), w)          # C not a multiple of 8
    assert e.value.status == gla.GTR_ERR_UNSUPPORTED
    G = torch.zeros((1, 4, 4, 16), dtype=torch.float16, device=dev)
    U = torch.zeros_like(G)
    w = torch.zeros((16, 3, 3), dtype=torch.float32, device=dev)
    with pytest.raises(gla.GTRError) as e:
        gla.gtr_spatial_swiglu_gate(G, U, w, out=U)         # out over U
    assert e.value.status == gla.GTR_ERR_INVALID_ARG
    empty = torch.zeros((1, 0, 4, 16), dtype=torch.float16, device=dev)
    gla.gtr_spatial_swiglu_gate(empty, empty.clone(), w)    # nothing to do
    assert gla.device_status() == gla.GTR_OK
    # silu(200) * 9 * 100 overflows fp16: reported, not returned silently
    G = torch.full((1, 4, 4, 16), 200.0, dtype=torch.float16, device=dev)
    U = torch.full((1, 4, 4, 16), 100.0, dtype=torch.float16, device=dev)
    w = torch.ones((16, 3, 3), dtype=torch.float32, device=dev)
    gla.gtr_spatial_swiglu_gate(G, U, w)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_ERR_RANGE
    assert gla.device_status() == gla.GTR_OK
