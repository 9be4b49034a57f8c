"""gtr_gla_fwd_stack: the 12-block direction-cycling stack as one recorded graph (GPU only).

The 768px batched workload (B=8, 16 heads, 48x48 grid) runs as twelve layer calls that
cycle L->R, R->L, T->B, B->T with fresh inputs per call.  Through the stack entry point
every layer's output must equal the same call made alone, bit for bit (same kernel, same
launch plan), on the first call (graph recorded) and on a repeat (graph replayed); the
layers checked against the fp64 oracle cover all four directions.  A chained stack (each
layer starting from the previous one's final state) must equal one long scan.
"""
import pytest
import torch

from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import DIR_NAMES, WORKLOADS, make_inputs, workload_inputs
from tests.gpu_common import assert_parity, run_oracle

pytestmark = pytest.mark.gpu


def test_twelve_layer_stack_matches_single_calls_and_oracle():
    w = WORKLOADS["b8h16_48x48_stack12"]
    dev = torch.device("cuda", 0)
    dirs = w.call_directions()
    assert len(dirs) == 12
    host = [workload_inputs(w, d, call) for call, d in enumerate(dirs)]
    layers = []
    for inp, d in zip(host, dirs):
        t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
        layers.append(dict(t, direction=d, final_state=True))
    for rep in range(2):   # recorded, then replayed
        res = gla.gtr_gla_fwd_stack(layers, w.H, w.W)
        torch.cuda.synchronize()
        assert gla.device_status() == gla.GTR_OK
        for i, (L, (out, fs)) in enumerate(zip(layers, res)):
            o1, s1 = gla.gtr_gla_fwd(L["q"], L["k"], L["v"], L["g"], w.H, w.W, L["direction"],
                                     final_state=True)
            torch.cuda.synchronize()
            assert torch.equal(out, o1), f"rep {rep} layer {i} out"
            assert torch.equal(fs, s1), f"rep {rep} layer {i} final state"
    for i in (0, 1, 2, 3, 11):   # every direction against the oracle
        ro, rs = run_oracle(host[i], w.H, w.W, dirs[i])
        out, fs = res[i]
        assert_parity(out.float().cpu().numpy(), ro, f"layer {i} {DIR_NAMES[dirs[i]]} out")
        assert_parity(fs.cpu().numpy(), rs, f"layer {i} {DIR_NAMES[dirs[i]]} final state")


def test_chained_stack_equals_one_long_scan():
    """Layer i+1 starts from layer i's final state: four layers over four row bands of a
    grid, L->R, equal one L->R call over the whole grid."""
    B, heads, H, W = 1, 3, 32, 24
    inp = make_inputs(B, heads, H, W, 64, 64, seed=55, init_std=0.2)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    band = H // 4 * W
    states = [inp["s0"].to(dev)] + [torch.empty((B, heads, 64, 64), device=dev) for _ in range(4)]
    layers = []
    for i in range(4):
        sl = {n: x[:, i * band:(i + 1) * band].contiguous() for n, x in t.items()}
        layers.append(dict(sl, direction=0, init_state=states[i], final_state=states[i + 1]))
    res = gla.gtr_gla_fwd_stack(layers, H // 4, W)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    ro, rs = run_oracle(inp, H, W, 0)
    out = torch.cat([o for o, _ in res], dim=1).float().cpu().numpy()
    assert_parity(out, ro, "chained out")
    assert_parity(states[4].cpu().numpy(), rs, "chained final state")


def test_wide_head_stack_matches_single_calls():
    """A four-layer stack with dk = dv = 128 (four launches per layer) equals the same
    calls made one by one, bit for bit."""
    B, heads, H, W = 1, 2, 20, 20
    dev = torch.device("cuda", 0)
    layers = []
    for i in range(4):
        inp = make_inputs(B, heads, H, W, 128, 128, seed=70 + i, init_std=0.2)
        t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
        layers.append(dict(t, direction=i, init_state=inp["s0"].to(dev), final_state=True))
    res = gla.gtr_gla_fwd_stack(layers, H, W)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    for i, (L, (out, fs)) in enumerate(zip(layers, res)):
        o1, s1 = gla.gtr_gla_fwd(L["q"], L["k"], L["v"], L["g"], H, W, L["direction"],
                                 init_state=L["init_state"], final_state=True)
        torch.cuda.synchronize()
        assert torch.equal(out, o1) and torch.equal(fs, s1), f"layer {i}"


def test_stack_argument_checks():
    dev = torch.device("cuda", 0)
    inp = make_inputs(1, 1, 4, 4, 64, 64, seed=1)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    with pytest.raises(gla.GTRError) as e:
        gla.gtr_gla_fwd_stack([dict(t, direction=5)], 4, 4)
    assert e.value.status == gla.GTR_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        q2 = torch.zeros((1, 16, 2, 64), dtype=torch.float16, device=dev)
        gla.gtr_gla_fwd_stack([dict(t, direction=0), dict(q=q2, k=q2, v=q2, g=q2, direction=0)], 4, 4)
    assert gla.device_status() == gla.GTR_OK
