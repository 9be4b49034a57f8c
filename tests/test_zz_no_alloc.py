"""gtr_gla_fwd_static (workspace in the library's static device scratch) against
gtr_gla_fwd, through the C ABI (GPU only).  Collected last on purpose: it must pass
both alone and after every other test has used the device."""
import pytest
import torch

from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import WORKLOADS, make_inputs, workload_inputs
from tests.gpu_common import MAX_REL, MEAN_REL, err_ratios

pytestmark = pytest.mark.gpu


def _close(got, ref, what):
    mx, mn, _ = err_ratios(got.float().cpu().numpy(), ref.float().cpu().numpy())
    assert mx <= MAX_REL and mn <= MEAN_REL, f"{what}: max {mx:.3e} mean {mn:.3e}"


def test_static_scratch_two_calls_match_default():
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
        _close(o1, o2, f"call {call} out")
        _close(s1, s2, f"call {call} state")


def test_static_scratch_rejects_oversized_plans(monkeypatch):
    # 148 sequences forced into 2 spans: the plan's workspace exceeds the static scratch
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "2")
    B, heads, H, W = 4, 37, 16, 16
    assert gla.workspace_bytes(B, heads, H, W, 64, 64) > gla.STATIC_WS_BYTES
    inp = make_inputs(B, heads, H, W, 64, 64, seed=3)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    with pytest.raises(gla.GTRError) as e:
        gla.gtr_gla_fwd_static(t["q"], t["k"], t["v"], t["g"], H, W, 0)
    assert e.value.status == gla.GTR_ERR_UNSUPPORTED
    assert gla.device_status() == gla.GTR_OK
