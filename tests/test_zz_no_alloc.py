"""gtr_gla_fwd_static (workspace in the library's static device scratch) against
gtr_gla_fwd, through the C ABI (GPU only).  Collected last on purpose: it must pass
both alone and after every other test has used the device."""
import pytest
import torch

from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import WORKLOADS, make_inputs, workload_inputs
from tests.gpu_common import assert_parity, run_oracle

pytestmark = pytest.mark.gpu


def test_static_scratch_two_calls_match_default():
    """Two calls in a row through the static scratch equal the default path bit for bit
    (same launch plan, deterministic kernel)."""
    w = WORKLOADS["gtr640_b1h16_40x40"]   # 16 sequences: spans exchange through the scratch
    assert gla.workspace_bytes(w.B, w.heads, w.H, w.W, w.dk, w.dv) > 0
    dev = torch.device("cuda", 0)
    for call, d in enumerate((1, 2)):
        inp = workload_inputs(w, d, 60 + call)
        t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
        o1, s1 = gla.gtr_gla_fwd_static(t["q"], t["k"], t["v"], t["g"], w.H, w.W, d,
                                         final_state=True)
        o2, s2 = gla.gtr_gla_fwd(t["q"], t["k"], t["v"], t["g"], w.H, w.W, d, final_state=True)
        torch.cuda.synchronize()
        assert gla.device_status() == gla.GTR_OK
        assert torch.equal(o1, o2), f"call {call} out"
        assert torch.equal(s1, s2), f"call {call} state"


def test_static_scratch_plans_within_its_size(monkeypatch):
    """148 sequences forced into 2 spans need more workspace than the scratch holds:
    the static call takes a plan that fits (one span per sequence) and stays exact."""
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "2")
    B, heads, H, W = 4, 37, 16, 16
    assert gla.workspace_bytes(B, heads, H, W, 64, 64) > gla.STATIC_WS_BYTES
    inp = make_inputs(B, heads, H, W, 64, 64, seed=3, init_std=0.2)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    out, sf = gla.gtr_gla_fwd_static(t["q"], t["k"], t["v"], t["g"], H, W, 0,
                                     init_state=inp["s0"].to(dev), final_state=True)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    ro, rs = run_oracle(inp, H, W, 0)
    assert_parity(out.float().cpu().numpy(), ro, "out")
    assert_parity(sf.cpu().numpy(), rs, "final state")


@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128), (128, 128)])
def test_static_scratch_wide_heads_match_default(dk, dv):
    """dk and / or dv = 128 (two or four launches over 64-wide halves) through the
    static scratch equal the default path bit for bit, and the oracle."""
    B, heads, H, W = 1, 4, 24, 24
    inp = make_inputs(B, heads, H, W, dk, dv, seed=dk + dv, init_std=0.3)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    s0 = inp["s0"].to(dev)
    o1, s1 = gla.gtr_gla_fwd_static(t["q"], t["k"], t["v"], t["g"], H, W, 3, init_state=s0, final_state=True)
    o2, s2 = gla.gtr_gla_fwd(t["q"], t["k"], t["v"], t["g"], H, W, 3, init_state=s0, final_state=True)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    ro, rs = run_oracle(inp, H, W, 3)
    assert_parity(o1.float().cpu().numpy(), ro, "out")
    assert_parity(s1.cpu().numpy(), rs, "final state")
