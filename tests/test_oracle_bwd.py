"""Pins of the oracle's backward pass (CPU only).

The backward (``oracle.gla_backward``) is reverse-mode differentiation of the key-decay
recurrence (GTR news article, section "线性注意力到底在省什么"), over the four scan orders
(section "单向扫描的致命缺陷，以及GTR怎么补"); the pages print no backward, and train the
backbone by distillation (section "老师教学生，但只教最后一道题的答案").  Here it is held
against things other than itself:

* central finite differences of the pinned forward oracle, every input, every direction;
* float64 autograd through an independent token loop written with torch ops, on a scan
  long enough to cross the oracle's recompute segments;
* the decay-gradient identity: with b_t the running sum of g, the loss depends on g only
  through the b's, and d/d b_t of q_t e^{b_t} and k_t e^{-b_t} gives
      dg_r = sum_{t >= r} (q_t * dq_t - k_t * dk_t) + sum_j dS_f[:, j] * S_final[:, j];
* closed forms at a == 0 (only the current token survives) and a == 1 (causal linear
  attention by prefix sums);
* planted mistakes in a copy of the oracle's source, each caught by these pins.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from tests import restatements as R
from tests.test_oracle_pins import rand_case

SRC = os.path.join(os.path.dirname(oracle.__file__), "gla_oracle.c")


def _upstream(rng, q, v, with_dsf=True):
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    do = rng.standard_normal((B, N, heads, dv))
    dsf = rng.standard_normal((B, heads, dk, dv)) if with_dsf else None
    return do, dsf


def _loss(fwd, q, k, v, g, s0, do, dsf, H, W, d):
    o, sf = fwd(q, k, v, g, H, W, d, s0)
    val = float(np.sum(o * do))
    if dsf is not None:
        val += float(np.sum(sf * dsf))
    return val


def fd_gradients(fwd, q, k, v, g, s0, do, dsf, H, W, d, eps=1e-6):
    """Central differences of the loss for every element of q, k, v, g, s0."""
    args = [q, k, v, g, s0]
    grads = []
    for idx, arr in enumerate(args):
        num = np.zeros_like(arr)
        for mi in np.ndindex(arr.shape):
            hi = [x.copy() for x in args]
            lo = [x.copy() for x in args]
            hi[idx][mi] += eps
            lo[idx][mi] -= eps
            num[mi] = (_loss(fwd, *hi, do, dsf, H, W, d) - _loss(fwd, *lo, do, dsf, H, W, d)) / (2 * eps)
        grads.append(num)
    return grads


def max_gap(a, b):
    return float(np.max(np.abs(a - b)) / max(1.0, float(np.max(np.abs(b)))))


def check_fd(bwd, fwd, seed=0):
    """Worst gap between the backward and finite differences over small cases."""
    rng = np.random.default_rng(seed)
    worst = 0.0
    for (B, heads, H, W, dk, dv) in ((1, 1, 1, 4, 2, 3), (1, 2, 2, 3, 3, 2)):
        for d in range(4):
            q, k, v, g, s0 = rand_case(rng, B, heads, H, W, dk, dv)
            g = np.maximum(g, -3.0)   # keep every term visible to the differences
            do, dsf = _upstream(rng, q, v)
            num = fd_gradients(fwd, q, k, v, g, s0, do, dsf, H, W, d)
            got = bwd(q, k, v, g, do, H, W, d, s0, dsf)
            for x, y in zip((got[0], got[1], got[2], got[3], got[4]), num):
                worst = max(worst, max_gap(x, y))
    return worst


def torch_reference_grads(q, k, v, g, s0, do, dsf, H, W, d):
    """Gradients by float64 autograd through a plain token loop (torch ops only)."""
    t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, g, s0)]
    tq, tk, tv, tg, ts0 = t
    B, N, heads, dk = q.shape
    perm = R.scan_permutation(H, W, d)
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for h in range(heads):
            S = ts0[b, h]
            for p in range(N):
                n = int(perm[p])
                S = torch.exp(tg[b, n, h])[:, None] * S + torch.outer(tk[b, n, h], tv[b, n, h])
                loss = loss + torch.dot(tq[b, n, h] @ S, torch.tensor(do[b, n, h]))
            loss = loss + torch.sum(S * torch.tensor(dsf[b, h]))
    grads = torch.autograd.grad(loss, t)
    return [x.numpy() for x in grads]


def check_autograd(bwd, seed=3):
    rng = np.random.default_rng(seed)
    worst = 0.0
    # 150 positions: three of the oracle's 64-position recompute segments
    B, heads, H, W, dk, dv = 1, 2, 10, 15, 4, 3
    for d in (0, 3):
        q, k, v, g, s0 = rand_case(rng, B, heads, H, W, dk, dv, g_mode="sigmoid")
        do, dsf = _upstream(rng, q, v)
        ref = torch_reference_grads(q, k, v, g, s0, do, dsf, H, W, d)
        got = bwd(q, k, v, g, do, H, W, d, s0, dsf)
        for x, y in zip(got, ref):
            worst = max(worst, max_gap(x, y))
    return worst


def check_dg_identity(bwd, fwd, seed=5):
    rng = np.random.default_rng(seed)
    worst = 0.0
    B, heads, H, W, dk, dv = 2, 2, 9, 11, 5, 4
    for d in range(4):
        q, k, v, g, s0 = rand_case(rng, B, heads, H, W, dk, dv, g_mode="sigmoid")
        do, dsf = _upstream(rng, q, v)
        dq, dkk, _, dg, _ = bwd(q, k, v, g, do, H, W, d, s0, dsf)
        _, sf = fwd(q, k, v, g, H, W, d, s0)
        perm = R.scan_permutation(H, W, d)
        x = (q * dq - k * dkk)[:, perm]                    # scan order
        suffix = np.flip(np.cumsum(np.flip(x, axis=1), axis=1), axis=1)
        const = np.einsum("bhij,bhij->bhi", dsf, sf)        # [B, heads, dk]
        expect = np.empty_like(dg)
        expect[:, perm] = suffix + const[:, None, :, :]
        worst = max(worst, max_gap(dg, expect))
    return worst


def _bwd(q, k, v, g, do, H, W, d, s0=None, dsf=None, lib=None):
    return oracle.gla_backward(q, k, v, g, do, H, W, d, s0, dsf, lib=lib)


def _fwd(q, k, v, g, H, W, d, s0=None, lib=None):
    return oracle.gla_forward(q, k, v, g, H, W, d, s0, lib=lib)


def test_matches_central_differences():
    assert check_fd(_bwd, _fwd) < 1e-6


def test_matches_float64_autograd_across_segments():
    assert check_autograd(_bwd) < 1e-11


def test_decay_gradient_identity():
    assert check_dg_identity(_bwd, _fwd) < 1e-11


@pytest.mark.parametrize("d", range(4))
def test_all_forget_closed_form(d):
    """a == 0: S_t = k_t^T v_t, so o_t = (q_t . k_t) v_t and nothing flows between tokens."""
    rng = np.random.default_rng(7)
    B, heads, H, W, dk, dv = 1, 2, 3, 4, 3, 5
    q, k, v, _, s0 = rand_case(rng, B, heads, H, W, dk, dv)
    g = np.full_like(q, -1e4)   # exp underflows to exactly 0 in fp64
    do, dsf = _upstream(rng, q, v)
    dq, dkk, dvv, dg, ds0 = _bwd(q, k, v, g, do, H, W, d, s0, dsf)
    dov = np.einsum("bnhj,bnhj->bnh", do, v)[..., None]
    qk = np.einsum("bnhi,bnhi->bnh", q, k)[..., None]
    last = R.scan_permutation(H, W, d)[-1]
    e_dk = dov * q
    e_dv = qk * do
    e_dk[:, last] += np.einsum("bhij,bhj->bhi", dsf, v[:, last])
    e_dv[:, last] += np.einsum("bhi,bhij->bhj", k[:, last], dsf)
    assert max_gap(dq, dov * k) < 1e-13
    assert max_gap(dkk, e_dk) < 1e-13
    assert max_gap(dvv, e_dv) < 1e-13
    assert np.all(dg == 0.0) and np.all(ds0 == 0.0)


@pytest.mark.parametrize("d", range(4))
def test_all_retain_is_linear_attention_by_prefix_sums(d):
    """a == 1: S_t = S0 + sum_{s<=t} k_s^T v_s and G_t = dS_f + sum_{t'>=t} q_t'^T dO_t'."""
    rng = np.random.default_rng(8)
    B, heads, H, W, dk, dv = 2, 1, 4, 5, 4, 3
    q, k, v, _, s0 = rand_case(rng, B, heads, H, W, dk, dv)
    g = np.zeros_like(q)
    do, dsf = _upstream(rng, q, v)
    dq, dkk, dvv, dg, ds0 = _bwd(q, k, v, g, do, H, W, d, s0, dsf)
    perm = R.scan_permutation(H, W, d)
    Q, K, V, DO = q[:, perm], k[:, perm], v[:, perm], do[:, perm]
    kv = np.einsum("bnhi,bnhj->bnhij", K, V)
    S = s0[:, None] + np.cumsum(kv, axis=1)                     # S_t
    S_prev = np.concatenate([s0[:, None], S[:, :-1]], axis=1)   # S_{t-1}
    qdo = np.einsum("bnhi,bnhj->bnhij", Q, DO)
    G = dsf[:, None] + np.flip(np.cumsum(np.flip(qdo, axis=1), axis=1), axis=1)
    e = {
        "dq": np.einsum("bnhij,bnhj->bnhi", S, DO),
        "dk": np.einsum("bnhij,bnhj->bnhi", G, V),
        "dv": np.einsum("bnhi,bnhij->bnhj", K, G),
        "dg": np.einsum("bnhij,bnhij->bnhi", G, S_prev),
    }
    for name, got in (("dq", dq), ("dk", dkk), ("dv", dvv), ("dg", dg)):
        assert max_gap(got[:, perm], e[name]) < 1e-12, name
    assert max_gap(ds0, G[:, 0]) < 1e-12


def test_no_state_arguments_mean_zero():
    rng = np.random.default_rng(9)
    q, k, v, g, _ = rand_case(rng, 1, 2, 3, 5, 4, 4, g_mode="sigmoid")
    do, _ = _upstream(rng, q, v, with_dsf=False)
    zero = np.zeros((1, 2, 4, 4))
    a = _bwd(q, k, v, g, do, 3, 5, 2, None, None)
    b = _bwd(q, k, v, g, do, 3, 5, 2, zero, zero)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ------------------------------------------------------------------ planted mistakes
MUTANTS = {
    # dq read from the state before the token's own update
    "dq_uses_previous_state": ("sq_ += St[(long)i * dv + j] * dot[j];",
                               "sq_ += Sprev[(long)i * dv + j] * dot[j];"),
    # the token's own output term missing from G_t
    "own_output_term_dropped": ("G[(long)i * dv + j] += qt[i] * dot[j];",
                                "G[(long)i * dv + j] += 0.0 * qt[i] * dot[j];"),
    # chain rule through a = exp(g) forgotten
    "dg_without_a": ("dg[row * dk + i] = at * sa;", "dg[row * dk + i] = sa;"),
    # dg paired with the state after the update
    "dg_uses_current_state": ("sa += G[(long)i * dv + j] * Sprev[(long)i * dv + j];",
                              "sa += G[(long)i * dv + j] * St[(long)i * dv + j];"),
    # gradient carried to the previous position without the decay
    "carry_without_decay": ("G[(long)i * dv + j] *= a[i];", "G[(long)i * dv + j] *= 1.0;"),
    # dv contracted with q instead of k (transposed operand)
    "dv_uses_q": ("s += kt[i] * G[(long)i * dv + j];", "s += qt[i] * G[(long)i * dv + j];"),
    # checkpoints taken one position late (only scans longer than a segment see it)
    "checkpoint_off_by_one": ("if (p % kSeg == 0) memcpy(ck", "if (p % kSeg == 1 || p == 0) memcpy(ck"),
    # the final state's gradient dropped
    "final_state_gradient_dropped": ("if (dsf) memcpy(G, dsf", "if (0) memcpy(G, dsf"),
    # dk contracted with dO instead of v (wrong operand of the same shape)
    "dk_uses_dout": ("sk += G[(long)i * dv + j] * vt[j];", "sk += G[(long)i * dv + j] * dot[j];"),
}


def pins_detect(lib):
    def bwd(*a, **kw):
        return oracle.gla_backward(*a, lib=lib, **kw)

    fwd_lib = oracle._get()   # the committed forward (its own pins hold it)

    def fwd(*a, **kw):
        return oracle.gla_forward(*a, lib=fwd_lib, **kw)

    return (check_fd(bwd, fwd) > 1e-6 or check_autograd(bwd) > 1e-11
            or check_dg_identity(bwd, fwd) > 1e-11)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, name
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    out = str(tmp_path / "libmutant.so")
    oracle.compile_oracle(str(src), out)
    assert pins_detect(oracle.load_library(out)), name


def test_committed_oracle_passes_the_mutant_pins():
    assert not pins_detect(oracle._get())


def test_bad_arguments_are_rejected():
    rng = np.random.default_rng(10)
    q, k, v, g, _ = rand_case(rng, 1, 1, 2, 2, 2, 2)
    do = rng.standard_normal(v.shape)
    with pytest.raises(ValueError):
        _bwd(q, k, v, g, do[:, :3], 2, 2, 0)
    with pytest.raises(ValueError):
        _bwd(q, k, v, g, do, 2, 3, 0)
    with pytest.raises(RuntimeError):
        _bwd(q, k, v, g, do, 2, 2, 7)



@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("d", [0, 3])
@pytest.mark.parametrize("gates", ["strong", "zero_mixed", "zero_all"])
def test_chunked_restatement_agrees(chunk, d, gates):
    """The chunked algebra of the backward kernels (the zero-gate count form of the
    running log-decay, the per-pair path of very strongly forgetting channels, a partial
    last chunk) equals the position-by-position backward."""
    rng = np.random.default_rng(30 + chunk + d)
    B, heads, H, W, dk, dv = 1, 2, 9, 13, 8, 6
    q, k, v, g, s0 = rand_case(rng, B, heads, H, W, dk, dv, g_mode="sigmoid")
    if gates == "strong":
        g[..., :2] -= 4.0   # two channels decay by ~e^-260 over 64 positions
    elif gates == "zero_mixed":
        g[rng.random(g.shape) < 0.1] = -np.inf   # gates of exactly 0 between ordinary ones
    else:
        g[:] = -np.inf
    do, dsf = _upstream(rng, q, v)
    ref = _bwd(q, k, v, g, do, H, W, d, s0, dsf)
    got = R.chunkwise_backward(q, k, v, g, do, H, W, d, s0, dsf, chunk=chunk)
    for x, y in zip(got, ref):
        assert max_gap(x, y) < 1e-12
