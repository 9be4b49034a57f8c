"""Pins of the oracle's forget-gate step (CPU only): g = log(sigmoid(z)) / tau.

Each pin is a fact of the logistic function itself, not a retyping of the oracle's
formula:
  * log(sigmoid(0)) = -log 2;
  * log(sigmoid(z)) - log(sigmoid(-z)) = z (sigmoid(z) / sigmoid(-z) = e^z);
  * sigmoid(z) + sigmoid(-z) = 1;
  * log(sigmoid(z)) -> z as z -> -inf and -> -e^-z as z -> +inf (asymptotes, no
    overflow or cancellation at |z| in the hundreds or thousands);
  * agreement with exact rational-free high-precision values (Python's decimal at 50
    digits) on a spread of z;
  * g scales as 1/tau; g <= 0 everywhere.
A mistake of sign, of branch or of the tau scaling fails at least one of these.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle


def _ls_decimal(z: float) -> float:
    getcontext().prec = 50
    d = Decimal(z)
    return float(-(Decimal(1) + (-d).exp()).ln())


def test_log_sigmoid_at_zero():
    assert oracle.gate(np.array([0.0]), 1.0)[0] == pytest.approx(-np.log(2.0), abs=1e-16)


def test_log_sigmoid_odd_difference_identity():
    z = np.linspace(-60.0, 60.0, 481)
    lp, ln = oracle.gate(z, 1.0), oracle.gate(-z, 1.0)
    np.testing.assert_allclose(lp - ln, z, rtol=0, atol=1e-12)


def test_sigmoid_sum_rule():
    z = np.linspace(-30.0, 30.0, 241)
    s = np.exp(oracle.gate(z, 1.0)) + np.exp(oracle.gate(-z, 1.0))
    np.testing.assert_allclose(s, 1.0, rtol=0, atol=1e-15)


def test_asymptotes_without_overflow():
    neg = np.array([-50.0, -745.0, -1e4, -1e300])
    np.testing.assert_allclose(oracle.gate(neg, 1.0), neg, rtol=1e-15)
    pos = np.array([40.0, 100.0, 700.0])
    np.testing.assert_allclose(oracle.gate(pos, 1.0), -np.exp(-pos), rtol=1e-12)
    assert oracle.gate(np.array([1e4, 1e300]), 1.0).tolist() == [0.0, 0.0]
    assert np.all(np.isfinite(oracle.gate(np.array([-1e300, 1e300, -1e38]), 16.0)))


def test_high_precision_values():
    z = [-20.0, -7.25, -1.0, -0.125, 0.001, 0.5, 2.0, 9.0, 33.0]
    got = oracle.gate(np.array(z), 1.0)
    want = np.array([_ls_decimal(x) for x in z])
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)


def test_tau_scaling_and_sign():
    rng = np.random.default_rng(3)
    z = rng.normal(0.0, 5.0, 1000)
    g1 = oracle.gate(z, 1.0)
    for tau in (0.5, 16.0, 3.0):
        np.testing.assert_allclose(oracle.gate(z, tau), g1 / tau, rtol=1e-15, atol=0)
    assert np.all(g1 <= 0.0)


def test_bad_tau_is_rejected():
    with pytest.raises(RuntimeError):
        oracle.gate(np.zeros(3), 0.0)
    with pytest.raises(RuntimeError):
        oracle.gate(np.zeros(3), -1.0)


def test_forward_with_gate_equals_forward_with_its_log_decay():
    """gla_forward_z is gla_forward fed the fp64 gate: the same recurrence."""
    rng = np.random.default_rng(5)
    B, N, heads, dk, dv = 1, 12, 2, 4, 3
    q, k = rng.normal(size=(B, N, heads, dk)), rng.normal(size=(B, N, heads, dk))
    v, z = rng.normal(size=(B, N, heads, dv)), rng.normal(size=(B, N, heads, dk))
    o1, s1 = oracle.gla_forward_z(q, k, v, z, 16.0, 3, 4, 2)
    o2, s2 = oracle.gla_forward(q, k, v, oracle.gate(z, 16.0), 3, 4, 2)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


GATE_MUTANTS = {
    # log1p(exp(+z)): the sign of the exponent flipped
    "exp_sign": ("log1p(exp(-fabs(x)))", "log1p(exp(fabs(x)))"),
    # the min(z, 0) branch dropped
    "branch_dropped": ("(x < 0.0 ? x : 0.0) - log1p", "0.0 - log1p"),
    # tau multiplies instead of dividing
    "tau_inverted": ("g[i] = ls / tau;", "g[i] = ls * tau;"),
}


@pytest.mark.parametrize("name", sorted(GATE_MUTANTS))
def test_planted_gate_mistake_is_caught(name, tmp_path):
    import os
    src_path = os.path.join(os.path.dirname(oracle.__file__), "gla_oracle.c")
    old, new = GATE_MUTANTS[name]
    text = open(src_path).read()
    assert text.count(old) == 1
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = oracle.load_library(oracle.compile_oracle(str(src), str(tmp_path / "libmutant.so")))
    z = np.linspace(-30.0, 30.0, 121)
    caught = False
    try:
        g1 = oracle.gate(z, 1.0, lib=lib)
        caught |= not np.allclose(g1 - oracle.gate(-z, 1.0, lib=lib), z, atol=1e-9)
        caught |= not np.allclose(oracle.gate(z, 16.0, lib=lib), g1 / 16.0, rtol=1e-12)
        caught |= abs(oracle.gate(np.array([0.0]), 1.0, lib=lib)[0] + np.log(2.0)) > 1e-12
        caught |= not np.allclose(np.exp(g1) + np.exp(oracle.gate(-z, 1.0, lib=lib)), 1.0, atol=1e-12)
    except (RuntimeError, FloatingPointError):
        caught = True
    assert caught, f"pins did not catch gate mutant {name}"
