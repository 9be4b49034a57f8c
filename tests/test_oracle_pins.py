"""Pins for the fp64 oracle (CPU only).

The pages print no worked example of the token mixer, so the oracle is pinned
to mathematics: an O(N^2) closed form, exact rational arithmetic, the a == 1
and a == 0 special cases, direction identities, chunk-size invariance of an
independent chunked restatement, state passing across a split, and linearity.
``tests/test_oracle_mutants.py`` shows that each planted mistake fails one of
these pins.
"""
from fractions import Fraction
import math

import numpy as np
import pytest

import oracle
from tests import restatements as R

DIRS = (0, 1, 2, 3)


def rand_case(rng, B, heads, H, W, dk, dv, g_scale=1.0, with_s0=True, g_mode="mixed"):
    N = H * W
    q = rng.standard_normal((B, N, heads, dk))
    k = rng.standard_normal((B, N, heads, dk))
    v = rng.standard_normal((B, N, heads, dv))
    if g_mode == "mixed":
        # log-decays from ~0 down to strongly forgetting, incl. a few very negative
        g = -np.abs(rng.standard_normal((B, N, heads, dk))) * g_scale
        g[rng.random(g.shape) < 0.05] = -30.0
    else:
        g = np.log(1.0 / (1.0 + np.exp(-rng.standard_normal((B, N, heads, dk))))) / 16.0
    s0 = rng.standard_normal((B, heads, dk, dv)) if with_s0 else None
    return q, k, v, g, s0


def rel_err(a, b):
    scale = max(np.max(np.abs(b)), 1e-300)
    return np.max(np.abs(a - b)) / scale


def check_brute_force(fwd, shapes=((1, 1, 1, 1, 2, 2), (1, 2, 1, 7, 4, 2), (2, 1, 3, 5, 2, 4),
                                   (1, 1, 5, 3, 8, 4), (1, 2, 4, 4, 4, 8))):
    """P1: oracle == closed form, every direction, with and without S0."""
    rng = np.random.default_rng(1)
    worst = 0.0
    for (B, heads, H, W, dk, dv) in shapes:
        for d in DIRS:
            for with_s0 in (False, True):
                q, k, v, g, s0 = rand_case(rng, B, heads, H, W, dk, dv, with_s0=with_s0)
                o, sf = fwd(q, k, v, g, H, W, d, s0)
                ob, sb = R.brute_force(q, k, v, g, H, W, d, s0)
                worst = max(worst, rel_err(o, ob), rel_err(sf, sb))
    return worst


def oracle_fwd(q, k, v, g, H, W, d, s0=None):
    return oracle.gla_forward(q, k, v, g, H, W, d, s0)


def test_scan_map_matches_grid_flips():
    for H, W in ((1, 1), (1, 9), (9, 1), (3, 5), (5, 3), (4, 4), (37, 53)):
        for d in DIRS:
            perm = R.scan_permutation(H, W, d)
            got = np.array([oracle.scan_to_token(p, H, W, d) for p in range(H * W)])
            assert np.array_equal(got, perm), (H, W, d)
            assert np.array_equal(np.sort(got), np.arange(H * W))


def test_brute_force_closed_form():
    assert check_brute_force(oracle_fwd) < 1e-12


def test_exact_rational_case():
    """Hand-sized case in exact rational arithmetic: a in {1, 3/4, 1/2, 1/4}."""
    H, W, dk, dv = 2, 2, 2, 3
    N = H * W
    a = [[Fraction(1, 2), Fraction(1)], [Fraction(3, 4), Fraction(1, 4)],
         [Fraction(1), Fraction(1, 2)], [Fraction(1, 4), Fraction(3, 4)]]
    qv = [[1, -2], [3, 1], [-1, 2], [2, 2]]
    kv = [[2, 1], [-1, 1], [1, 3], [0, -2]]
    vv = [[1, 0, -1], [2, 1, 0], [-3, 1, 1], [1, 1, 1]]
    s0 = [[Fraction(1, 2), 0, 1], [2, Fraction(-1, 3), 0]]
    for d in DIRS:
        perm = R.scan_permutation(H, W, d)
        # exact recurrence in scan order, written as explicit sums of products
        exp_out = {}
        for t in range(N):
            acc = [Fraction(0)] * dv
            for s in range(t + 1):
                for i in range(dk):
                    w = Fraction(1)
                    for r in range(s + 1, t + 1):
                        w *= a[perm[r]][i]
                    c = Fraction(qv[perm[t]][i]) * w * kv[perm[s]][i]
                    for j in range(dv):
                        acc[j] += c * vv[perm[s]][j]
            for i in range(dk):
                w = Fraction(1)
                for r in range(t + 1):
                    w *= a[perm[r]][i]
                for j in range(dv):
                    acc[j] += Fraction(qv[perm[t]][i]) * w * Fraction(s0[i][j])
            exp_out[perm[t]] = acc
        q = np.array(qv, float).reshape(1, N, 1, dk)
        k = np.array(kv, float).reshape(1, N, 1, dk)
        v = np.array(vv, float).reshape(1, N, 1, dv)
        g = np.array([[math.log(x) for x in row] for row in a]).reshape(1, N, 1, dk)
        S0 = np.array([[float(x) for x in row] for row in s0]).reshape(1, 1, dk, dv)
        o, _ = oracle.gla_forward(q, k, v, g, H, W, d, S0)
        for n in range(N):
            for j in range(dv):
                assert abs(o[0, n, 0, j] - float(exp_out[n][j])) <= 1e-13 * (
                    1 + abs(float(exp_out[n][j]))), (d, n, j)


@pytest.mark.parametrize("d", DIRS)
def test_all_retain_is_causal_linear_attention(d):
    """P2: g == 0 (a == 1) reduces to causal linear attention."""
    rng = np.random.default_rng(2)
    q, k, v, _, s0 = rand_case(rng, 2, 2, 5, 7, 8, 4)
    g = np.zeros_like(q)
    o, sf = oracle.gla_forward(q, k, v, g, 5, 7, d, s0)
    ol, sl = R.linear_attention_prefix(q, k, v, 5, 7, d, s0)
    assert rel_err(o, ol) < 1e-12 and rel_err(sf, sl) < 1e-12


@pytest.mark.parametrize("g_value", [-np.inf, -1e4])
@pytest.mark.parametrize("d", DIRS)
def test_all_forget_keeps_only_current_token(d, g_value):
    """P3: a == 0: o_t = (q_t . k_t) v_t, final state = k_last^T v_last."""
    rng = np.random.default_rng(3)
    H, W = 4, 6
    q, k, v, _, s0 = rand_case(rng, 1, 3, H, W, 4, 5)
    g = np.full_like(q, g_value)
    o, sf = oracle.gla_forward(q, k, v, g, H, W, d, s0)
    expect = np.einsum("bnhi,bnhi->bnh", q, k)[..., None] * v
    assert rel_err(o, expect) < 1e-14
    last = R.scan_permutation(H, W, d)[-1]
    assert rel_err(sf, np.einsum("bhi,bhj->bhij", k[:, last], v[:, last])) < 1e-14


def test_direction_identities():
    """P4: R->L and B->T are the mirrored grids; T->B is the transposed grid."""
    rng = np.random.default_rng(4)
    B, heads, H, W, dk, dv = 2, 2, 4, 6, 4, 3
    q, k, v, g, s0 = rand_case(rng, B, heads, H, W, dk, dv)

    def grid(x):
        return x.reshape(B, H, W, heads, -1)

    def flat(x):
        return np.ascontiguousarray(x).reshape(B, -1, heads, x.shape[-1])

    # R->L == L->R on the horizontally mirrored grid
    mir = [flat(grid(t)[:, :, ::-1]) for t in (q, k, v, g)]
    o_m, s_m = oracle.gla_forward(*mir, H, W, 0, s0)
    o_r, s_r = oracle.gla_forward(q, k, v, g, H, W, 1, s0)
    assert rel_err(o_r, flat(grid(o_m)[:, :, ::-1])) < 1e-13 and rel_err(s_r, s_m) < 1e-13
    # B->T == T->B on the vertically mirrored grid
    mir = [flat(grid(t)[:, ::-1]) for t in (q, k, v, g)]
    o_m, s_m = oracle.gla_forward(*mir, H, W, 2, s0)
    o_b, s_b = oracle.gla_forward(q, k, v, g, H, W, 3, s0)
    assert rel_err(o_b, flat(grid(o_m)[:, ::-1])) < 1e-13 and rel_err(s_b, s_m) < 1e-13
    # T->B on H x W == L->R on the transposed W x H grid
    tr = [flat(grid(t).transpose(0, 2, 1, 3, 4)) for t in (q, k, v, g)]
    o_t, s_t = oracle.gla_forward(*tr, W, H, 0, s0)
    o_c, s_c = oracle.gla_forward(q, k, v, g, H, W, 2, s0)
    back = flat(o_t.reshape(B, W, H, heads, dv).transpose(0, 2, 1, 3, 4))
    assert rel_err(o_c, back) < 1e-13 and rel_err(s_c, s_t) < 1e-13


@pytest.mark.parametrize("chunk", [1, 16, 32, 64])
@pytest.mark.parametrize("g_mode", ["mixed", "logsigmoid"])
def test_chunk_size_invariance(chunk, g_mode):
    """P5: the chunked restatement equals the token-by-token oracle for any chunk."""
    rng = np.random.default_rng(5 + chunk)
    H, W = 9, 15          # 135 tokens: two full 64-chunks + a 7-token tail
    q, k, v, g, s0 = rand_case(rng, 1, 2, H, W, 8, 4, g_scale=0.3, g_mode=g_mode)
    for d in DIRS:
        o, sf = oracle.gla_forward(q, k, v, g, H, W, d, s0)
        oc, sc = R.chunkwise(q, k, v, g, H, W, d, s0, chunk=chunk)
        assert rel_err(oc, o) < 1e-10 and rel_err(sc, sf) < 1e-10, d


@pytest.mark.parametrize("m", [0, 1, 17, 64, 100, 134, 135])
def test_state_passing_split(m):
    """P6: running [0, m) then [m, N) from the carried state equals the full run."""
    rng = np.random.default_rng(6)
    H, W = 9, 15
    q, k, v, g, s0 = rand_case(rng, 2, 2, H, W, 4, 3)
    for d in DIRS:
        o, sf = oracle.gla_forward(q, k, v, g, H, W, d, s0)
        o1, s1 = oracle.gla_forward(q, k, v, g, H, W, d, s0, p_begin=0, p_end=m)
        o2, s2 = oracle.gla_forward(q, k, v, g, H, W, d, s1, p_begin=m, out=o1.copy())
        assert rel_err(o2, o) < 1e-13 and rel_err(s2, sf) < 1e-13


def test_linearity():
    """P7: linear in v at S0 = 0, and linear in S0 at v = 0."""
    rng = np.random.default_rng(7)
    H, W = 5, 6
    q, k, v1, g, s0 = rand_case(rng, 1, 2, H, W, 4, 3)
    v2 = rng.standard_normal(v1.shape)
    for d in DIRS:
        a, sa = oracle.gla_forward(q, k, v1, g, H, W, d)
        b, sb = oracle.gla_forward(q, k, v2, g, H, W, d)
        c, sc = oracle.gla_forward(q, k, 2.0 * v1 - 3.0 * v2, g, H, W, d)
        assert rel_err(c, 2 * a - 3 * b) < 1e-12 and rel_err(sc, 2 * sa - 3 * sb) < 1e-12
        z = np.zeros_like(v1)
        e, se = oracle.gla_forward(q, k, z, g, H, W, d, s0)
        f, sf_ = oracle.gla_forward(q, k, z, g, H, W, d, -0.5 * s0)
        assert rel_err(f, -0.5 * e) < 1e-13 and rel_err(sf_, -0.5 * se) < 1e-13


def test_empty_grid_and_bad_args():
    q = np.zeros((1, 0, 2, 4))
    v = np.zeros((1, 0, 2, 3))
    o, sf = oracle.gla_forward(q, q, v, q, 0, 5, 0)
    assert o.shape == (1, 0, 2, 3) and not sf.any()
    with pytest.raises(ValueError):
        oracle.gla_forward(np.zeros((1, 6, 1, 2)), np.zeros((1, 6, 1, 2)),
                           np.zeros((1, 6, 1, 2)), np.zeros((1, 6, 1, 2)), 2, 2, 0)
    with pytest.raises(RuntimeError):
        z = np.zeros((1, 4, 1, 2))
        oracle.gla_forward(z, z, z, z, 2, 2, 7)
