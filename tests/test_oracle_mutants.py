"""Planted mistakes in the oracle must fail at least one pin (CPU only).

Each mutant is a textual edit of a temporary copy of ``oracle/gla_oracle.c``,
compiled into a temporary library; the committed oracle is never touched.
"""
import os

import numpy as np
import pytest

import oracle
from tests import restatements as R
from tests.test_oracle_pins import check_brute_force, rand_case, rel_err

SRC = os.path.join(os.path.dirname(oracle.__file__), "gla_oracle.c")

MUTANTS = {
    # decay applied after the current token's k v is added (wrong product range)
    "decay_after_update": ("a[i] * S[(long)i * dv + j] + kt[i] * vt[j]",
                           "a[i] * (S[(long)i * dv + j] + kt[i] * vt[j])"),
    # value-side decay instead of key-side decay (transposed operand)
    "value_side_decay": ("a[i] * S[(long)i * dv + j]", "a[j % dk] * S[(long)i * dv + j]"),
    # sign error in the gate
    "gate_sign": ("a[i] = exp(gt[i])", "a[i] = exp(-gt[i])"),
    # dropped initial-state term
    "dropped_s0": ("if (s0)\n", "if (0)\n"),
    # R->L read as L->R
    "r2l_not_mirrored": ("case DIR_R2L: y = p / W; x = W - 1 - p % W;",
                         "case DIR_R2L: y = p / W; x = p % W;"),
    # B->T read as T->B
    "b2t_not_mirrored": ("default:      x = p / H; y = H - 1 - p % H;",
                         "default:      x = p / H; y = p % H;"),
    # T->B with the roles of H and W swapped
    "t2b_swapped": ("case DIR_T2B: x = p / H; y = p % H;",
                    "case DIR_T2B: y = p / W; x = p % W;"),
    # output read with k instead of q
    "output_uses_k": ("acc += qt[i] * S", "acc += kt[i] * S"),
}


def pins_detect(lib):
    def fwd(q, k, v, g, H, W, d, s0=None, **kw):
        return oracle.gla_forward(q, k, v, g, H, W, d, s0, lib=lib, **kw)

    if check_brute_force(fwd) > 1e-9:
        return True
    rng = np.random.default_rng(11)
    q, k, v, g, s0 = rand_case(rng, 1, 2, 4, 6, 4, 3)
    for d in range(4):
        o, _ = fwd(q, k, v, g, 4, 6, d, s0)
        oc, _ = R.chunkwise(q, k, v, g, 4, 6, d, s0, chunk=16)
        if rel_err(o, oc) > 1e-9:
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    so = oracle.compile_oracle(str(src), str(tmp_path / "libmutant.so"))
    assert pins_detect(oracle.load_library(so)), f"pins did not catch mutant {name}"


def test_unmutated_copy_passes(tmp_path):
    src = tmp_path / "same.c"
    src.write_text(open(SRC).read())
    so = oracle.compile_oracle(str(src), str(tmp_path / "libsame.so"))
    assert not pins_detect(oracle.load_library(so))
