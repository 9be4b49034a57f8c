"""Device-side failure path (GPU only), without faulting the GPU.

Every wait in the kernels is bounded; a wait that runs out sets the device error
word, the kernel ends normally and gtr_gla_device_status reports GTR_ERR_TIMEOUT.
The library's self-test kernel makes its waits run out on purpose (a barrier that
nothing arrives on, a flag that nothing sets, a short limit) through the same
bounded-wait code; the context must stay usable afterwards.
"""
import pytest
import torch

from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import WORKLOADS, workload_inputs
from tests.gpu_common import assert_parity, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def test_selftest_timeout_is_reported_then_cleared():
    torch.cuda.init()
    assert gla.device_status() == gla.GTR_OK
    assert gla.selftest_timeout(2000) == gla.GTR_OK
    assert gla.device_status() == gla.GTR_ERR_TIMEOUT
    assert gla.device_status() == gla.GTR_OK   # read and cleared


def test_selftest_limit_is_checked():
    assert gla.selftest_timeout(0) == gla.GTR_ERR_INVALID_ARG
    assert gla.selftest_timeout(2_000_000) == gla.GTR_ERR_INVALID_ARG
    assert gla.device_status() == gla.GTR_OK   # nothing was launched


def test_span_call_after_a_timeout_matches_the_oracle():
    """After a reported timeout the library zero-fills its workspaces; a span call
    (several CTAs per sequence exchanging aggregates) is exact again."""
    w = WORKLOADS["gtr640_b1h16_40x40"]
    assert gla.plan(w.B, w.heads, w.H, w.W, w.dk, w.dv)[0] > 1
    out, _ = run_gpu(workload_inputs(w, 0, 70), w.H, w.W, 0)   # the cached workspace exists
    assert gla.selftest_timeout(1000) == gla.GTR_OK
    assert gla.device_status() == gla.GTR_ERR_TIMEOUT
    inp = workload_inputs(w, 2, 71)
    out, st = run_gpu(inp, w.H, w.W, 2)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    ro, rs = run_oracle(inp, w.H, w.W, 2)
    assert_parity(out, ro, "out after timeout")
    assert_parity(st, rs, "state after timeout")
