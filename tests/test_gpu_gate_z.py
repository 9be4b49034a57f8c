"""Gate fused into the kernel: gtr_gla_fwd_z (z and tau in place of g) vs the fp64 oracle
fed the oracle's own fp64 gate g = log(sigmoid(z)) / tau (GPU only).

The z draws follow the workloads' recipe (z ~ N(0, 1), tau = 16) at every dk = 64
workload and direction, plus temperatures other than 16 and pre-activations up to
|z| = 60 (gates that are 1 or 0 to working precision), with spans forced so that the
look-back and the corrections see the fused gate too.
"""
import pytest
import torch

import oracle
from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import WORKLOADS, make_inputs
from tests.gpu_common import assert_parity

pytestmark = pytest.mark.gpu


def _z_inputs(B, heads, H, W, seed, zscale=1.0, zshift=0.0, init_std=None):
    inp = make_inputs(B, heads, H, W, 64, 64, seed=seed, init_std=init_std)
    gen = torch.Generator().manual_seed(seed + 1)
    z = torch.randn((B, H * W, heads, 64), generator=gen) * zscale + zshift
    inp["z"] = z.half()
    return inp


def _run(inp, tau, H, W, d):
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "z")}
    s0 = None if inp.get("s0") is None else inp["s0"].to(dev)
    out, sf = gla.gtr_gla_fwd_z(t["q"], t["k"], t["v"], t["z"], tau, H, W, d, init_state=s0,
                                final_state=True)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    f = lambda x: x.float().numpy()  # noqa: E731
    s0n = None if inp.get("s0") is None else inp["s0"].numpy()
    ro, rs = oracle.gla_forward_z(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["z"]), tau, H, W, d,
                                  s0n)
    return out.float().cpu().numpy(), sf.cpu().numpy(), ro, rs


CASES = [(w.name, d) for w in WORKLOADS.values() if w.dk == 64 and w.calls == 1 for d in w.directions]


@pytest.mark.parametrize("name,direction", CASES)
def test_workloads_with_fused_gate(name, direction):
    w = WORKLOADS[name]
    inp = _z_inputs(w.B, w.heads, w.H, w.W, seed=700 + 10 * w.index + direction,
                    init_std=w.init_std)
    out, sf, ro, rs = _run(inp, 16.0, w.H, w.W, direction)
    assert_parity(out, ro, f"{name} out")
    assert_parity(sf, rs, f"{name} final state")


@pytest.mark.parametrize("tau,zscale,zshift", [(1.0, 1.0, 0.0), (4.0, 3.0, 1.0), (64.0, 1.0, -2.0),
                                               (16.0, 20.0, 0.0), (16.0, 1.0, 59.0),
                                               (16.0, 1.0, -59.0)])
@pytest.mark.parametrize("spans", [None, 5])
def test_temperatures_and_extreme_pre_activations(monkeypatch, tau, zscale, zshift, spans):
    if spans:
        monkeypatch.setenv("GTR_CLUSTER_SIZE", str(spans))
    B, heads, H, W = 1, 4, 40, 40
    inp = _z_inputs(B, heads, H, W, seed=811, zscale=zscale, zshift=zshift, init_std=0.3)
    for d in (0, 3):
        out, sf, ro, rs = _run(inp, tau, H, W, d)
        assert_parity(out, ro, f"tau {tau} z*{zscale}+{zshift} dir {d} out")
        assert_parity(sf, rs, f"tau {tau} z*{zscale}+{zshift} dir {d} final state")


def test_bad_temperature_is_rejected():
    dev = torch.device("cuda", 0)
    inp = _z_inputs(1, 1, 4, 4, seed=1)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "z")}
    for tau in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(gla.GTRError) as e:
            gla.gtr_gla_fwd_z(t["q"], t["k"], t["v"], t["z"], tau, 4, 4, 0)
        assert e.value.status == gla.GTR_ERR_INVALID_ARG
    assert gla.device_status() == gla.GTR_OK


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_dk128_with_fused_gate(direction):
    """dk = 128 (two 64-channel halves, the second adding to the first's output)."""
    B, heads, H, W = 2, 3, 19, 23
    inp = make_inputs(B, heads, H, W, 128, 64, seed=901 + direction, init_std=0.3)
    gen = torch.Generator().manual_seed(902 + direction)
    inp["z"] = (torch.randn((B, H * W, heads, 128), generator=gen) * 2.0).half()
    out, sf, ro, rs = _run(inp, 8.0, H, W, direction)
    assert_parity(out, ro, "dk128 out")
    assert_parity(sf, rs, "dk128 final state")


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 128)])
def test_wide_values_with_fused_gate(dk, dv):
    """dv = 128 (two value halves), with dk = 64 or 128, through the fused gate."""
    B, heads, H, W = 1, 3, 17, 29
    inp = make_inputs(B, heads, H, W, dk, dv, seed=930 + dk + dv, init_std=0.3)
    gen = torch.Generator().manual_seed(931)
    inp["z"] = (torch.randn((B, H * W, heads, dk), generator=gen) * 2.0).half()
    for d in (1, 2):
        out, sf, ro, rs = _run(inp, 16.0, H, W, d)
        assert_parity(out, ro, f"dk{dk} dv{dv} dir {d} out")
        assert_parity(sf, rs, f"dk{dk} dv{dv} dir {d} final state")
