"""Pins of the Spatial SwiGLU gated value branch in the oracle (CPU only):
h = silu(G) * (bias + 3x3 depthwise cross-correlation of U, zero padding).

Each pin is a fact fixed independently of the oracle's own loop:
  * SiLU: silu(0) = 0, silu(x) - silu(-x) = x, asymptotes, 50-digit values;
  * a kernel with a single tap at (i, j) moves U by (i-1, j-1) with zeros entering
    from the border (the orientation and the padding of the stencil);
  * random kernels against scipy's 2-D cross-correlation of each channel
    (``correlate2d``, zero fill, same size) — a library routine;
  * linearity in U, in w, and the bias term silu(G) * bias;
  * planted mistakes (convolution instead of cross-correlation, wrap-around
    padding, the sigmoid's sign, the bias dropped) each fail one of these.
"""
from decimal import Decimal, getcontext
import os

import numpy as np
import pytest
from scipy.signal import correlate2d

import oracle


def _silu_decimal(x: float) -> float:
    getcontext().prec = 50
    d = Decimal(x)
    return float(d / (Decimal(1) + (-d).exp()))


def test_silu_values_and_identities():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    x = np.linspace(-40.0, 40.0, 321)
    np.testing.assert_allclose(oracle.silu(x) - oracle.silu(-x), x, rtol=0, atol=1e-12)
    pts = [-30.0, -4.5, -1.0, -0.01, 0.25, 1.0, 3.0, 17.0]
    np.testing.assert_allclose(oracle.silu(np.array(pts)), [_silu_decimal(p) for p in pts], rtol=1e-14)
    np.testing.assert_allclose(oracle.silu(np.array([50.0, 700.0])), [50.0, 700.0], rtol=1e-15)
    assert abs(oracle.silu(np.array([-800.0]))[0]) < 1e-300


def _rand(shape, seed):
    return np.random.default_rng(seed).normal(size=shape)


@pytest.mark.parametrize("i,j", [(0, 0), (0, 2), (1, 1), (2, 0), (2, 1)])
def test_single_tap_shifts_with_zero_border(i, j):
    B, H, W, C = 2, 5, 7, 3
    G, U = _rand((B, H, W, C), 1), _rand((B, H, W, C), 2)
    w = np.zeros((C, 3, 3))
    w[:, i, j] = 1.0
    h = oracle.spatial_swiglu_gate(G, U, w)
    shifted = np.zeros_like(U)
    dy, dx = i - 1, j - 1   # output (y, x) reads U at (y + dy, x + dx)
    for y in range(H):
        for x in range(W):
            if 0 <= y + dy < H and 0 <= x + dx < W:
                shifted[:, y, x] = U[:, y + dy, x + dx]
    sig = 1.0 / (1.0 + np.exp(-G))
    np.testing.assert_allclose(h, G * sig * shifted, rtol=1e-13, atol=1e-15)


def test_random_kernels_match_library_cross_correlation():
    B, H, W, C = 2, 6, 9, 4
    G, U, w = _rand((B, H, W, C), 3), _rand((B, H, W, C), 4), _rand((C, 3, 3), 5)
    bias = _rand((C,), 6)
    h = oracle.spatial_swiglu_gate(G, U, w, bias)
    ref = np.empty_like(U)
    for b in range(B):
        for c in range(C):
            ref[b, :, :, c] = correlate2d(U[b, :, :, c], w[c], mode="same", boundary="fill") + bias[c]
    ref *= G / (1.0 + np.exp(-G))
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-13)


def test_linearity_and_bias():
    B, H, W, C = 1, 4, 4, 5
    G, U1, U2 = _rand((B, H, W, C), 7), _rand((B, H, W, C), 8), _rand((B, H, W, C), 9)
    w1, w2 = _rand((C, 3, 3), 10), _rand((C, 3, 3), 11)
    f = oracle.spatial_swiglu_gate
    np.testing.assert_allclose(f(G, U1 + U2, w1), f(G, U1, w1) + f(G, U2, w1), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(f(G, U1, w1 + w2), f(G, U1, w1) + f(G, U1, w2), rtol=1e-12, atol=1e-13)
    bias = _rand((C,), 12)
    np.testing.assert_allclose(f(G, U1, w1, bias) - f(G, U1, w1), oracle.silu(G) * bias, rtol=1e-12,
                               atol=1e-13)


MUTANTS = {
    # convolution (kernel flipped) instead of cross-correlation
    "flipped": ("w[c * 9 + i * 3 + j]", "w[c * 9 + (2 - i) * 3 + (2 - j)]"),
    # wrap-around instead of zero padding
    "wrap": ("if (yy < 0 || yy >= H || xx < 0 || xx >= W) continue;",
             "const long yw = (yy + H) % H, xw = (xx + W) % W; acc += w[c * 9 + i * 3 + j] * "
             "U[((b * H + yw) * W + xw) * C + c]; continue;"),
    # sigmoid of -x
    "sigmoid_sign": ("return x / (1.0 + exp(-x));", "return x / (1.0 + exp(x));"),
    # bias dropped
    "no_bias": ("double acc = bias ? bias[c] : 0.0;", "double acc = 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = os.path.join(os.path.dirname(oracle.__file__), "swiglu_oracle.c")
    old, new = MUTANTS[name]
    text = open(src).read()
    assert text.count(old) == 1
    p = tmp_path / "mutant.c"
    p.write_text(text.replace(old, new))
    lib = oracle.load_swiglu_library(oracle.compile_oracle(str(p), str(tmp_path / "libm.so")))
    caught = False
    # the pins above, run against the mutant
    x = np.linspace(-40.0, 40.0, 321)
    caught |= not np.allclose(oracle.silu(x, lib=lib) - oracle.silu(-x, lib=lib), x, atol=1e-9)
    B, H, W, C = 1, 5, 6, 3
    G, U, w = _rand((B, H, W, C), 21), _rand((B, H, W, C), 22), _rand((C, 3, 3), 23)
    bias = _rand((C,), 24)
    h = oracle.spatial_swiglu_gate(G, U, w, bias, lib=lib)
    ref = np.empty_like(U)
    for c in range(C):
        ref[0, :, :, c] = correlate2d(U[0, :, :, c], w[c], mode="same", boundary="fill") + bias[c]
    ref *= G / (1.0 + np.exp(-G))
    caught |= not np.allclose(h, ref, rtol=1e-9, atol=1e-9)
    assert caught, f"pins did not catch mutant {name}"
