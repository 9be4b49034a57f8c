"""CUDA path vs the fp64 oracle, element by element, through the C ABI (GPU only).

Every workload of the table in ``recurrent_vision_backbone_b200.inputs`` and all of
its scan directions run at full size, in the launch configuration the library
picks for that shape (the one bench.py times).  Edge cases cover ragged tails,
degenerate grids, the all-retain / all-forget gates, gates strong enough to
trigger the exact diagonal fallback, initial states and in-place carry.
"""
import numpy as np
import pytest
import torch

from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import DIR_NAMES, WORKLOADS, make_inputs, workload_inputs
from tests.gpu_common import assert_parity, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

CASES = []
for w in WORKLOADS.values():
    if w.calls > 1:
        # the stacked workload: 12 calls cycling the directions, fresh inputs per call
        for call, d in enumerate(w.call_directions()):
            CASES.append((w.name, d, call))
    else:
        for d in w.directions:
            CASES.append((w.name, d, 0))


@pytest.mark.parametrize("name,direction,call", CASES,
                         ids=[f"{n}-{DIR_NAMES[d]}-c{c}" for n, d, c in CASES])
def test_workload_parity(name, direction, call):
    w = WORKLOADS[name]
    inp = workload_inputs(w, direction, call)
    out, sf = run_gpu(inp, w.H, w.W, direction, final_state=True)
    ref_o, ref_s = run_oracle(inp, w.H, w.W, direction)
    assert_parity(out, ref_o, f"{name} {DIR_NAMES[direction]} out")
    assert_parity(sf, ref_s, f"{name} {DIR_NAMES[direction]} final state")


EDGE = [
    # B, heads, H, W, dk, init
    (1, 1, 1, 1, 64, False),      # one token
    (1, 2, 1, 77, 64, True),      # a single row: one full chunk + ragged tail
    (2, 1, 77, 1, 64, True),      # a single column
    (1, 3, 9, 15, 128, True),     # 135 tokens, dk = 128
    (3, 2, 8, 8, 64, False),      # exactly one chunk
    (1, 1, 13, 11, 128, False),   # 143 tokens: 2 chunks + 15-token tail
    (2, 5, 16, 16, 64, True),     # 4 chunks, 10 sequences
]


@pytest.mark.parametrize("B,heads,H,W,dk,init", EDGE)
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_edge_shapes(B, heads, H, W, dk, init, direction):
    inp = make_inputs(B, heads, H, W, dk, 64, seed=77 + H * 31 + W, init_std=0.5 if init else None)
    out, sf = run_gpu(inp, H, W, direction)
    ro, rs = run_oracle(inp, H, W, direction)
    assert_parity(out, ro, "out")
    assert_parity(sf, rs, "final state")


DV128 = [
    # B, heads, H, W, dk, init
    (1, 3, 9, 15, 64, True),      # dv = 128: two value-column halves
    (2, 1, 13, 11, 128, True),    # dk = dv = 128: four launches
    (1, 2, 40, 40, 64, False),    # 25 chunks: spans, look-back and corrections per half
]


@pytest.mark.parametrize("B,heads,H,W,dk,init", DV128)
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_dv128_shapes(B, heads, H, W, dk, init, direction):
    inp = make_inputs(B, heads, H, W, dk, 128, seed=97 + H * 31 + W + dk, init_std=0.5 if init else None)
    out, sf = run_gpu(inp, H, W, direction)
    ro, rs = run_oracle(inp, H, W, direction)
    assert_parity(out, ro, "out")
    assert_parity(sf, rs, "final state")


def test_dv128_in_place_carry():
    """init_state == final_state with dv = 128 (the halves carry disjoint columns)."""
    B, heads, H, W = 1, 2, 12, 10
    inp = make_inputs(B, heads, H, W, 128, 128, seed=13, init_std=0.2)
    dev = torch.device("cuda", 0)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "g"))
    st = inp["s0"].to(dev).clone()
    out, sf = gla.gtr_gla_fwd(q, k, v, g, H, W, 3, init_state=st, final_state=st)
    torch.cuda.synchronize()
    ro, rs = run_oracle(inp, H, W, 3)
    assert_parity(out.float().cpu().numpy(), ro, "out")
    assert_parity(st.cpu().numpy(), rs, "carried state")


@pytest.mark.parametrize("mode", ["retain", "forget_inf", "forget_big", "mixed_extreme",
                                  "strong"])
def test_degenerate_gates(mode):
    B, heads, H, W, dk = 1, 4, 20, 20, 64

    def z_of(shape):
        gen = torch.Generator().manual_seed(5)
        z = torch.randn(shape, generator=gen)
        if mode == "retain":
            return torch.full(shape, 60.0)            # logsigmoid(60)/16 == 0 in fp16
        if mode == "forget_inf":
            return torch.full(shape, -1e38)
        if mode == "forget_big":
            return torch.full(shape, -3000.0)         # g ~ -187: a == 0 in fp32
        if mode == "mixed_extreme":
            z = z * 40.0                              # mixes a ~ 1 and a ~ 0 within sub-blocks
            return z
        return z * 2.0 - 30.0                          # g ~ -1.9: diagonal fallback everywhere

    inp = make_inputs(B, heads, H, W, dk, 64, seed=9, init_std=0.3, z_override=z_of)
    for d in range(4):
        out, sf = run_gpu(inp, H, W, d)
        ro, rs = run_oracle(inp, H, W, d)
        assert_parity(out, ro, f"{mode} out dir {d}")
        assert_parity(sf, rs, f"{mode} state dir {d}")


def test_in_place_state_carry():
    """init_state == final_state: the call reads its state and overwrites it."""
    B, heads, H, W = 1, 3, 12, 10
    inp = make_inputs(B, heads, H, W, 64, 64, seed=3, init_std=0.2)
    dev = torch.device("cuda", 0)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "g"))
    st = inp["s0"].to(dev).clone()
    out, sf = gla.gtr_gla_fwd(q, k, v, g, H, W, 2, init_state=st, final_state=st)
    torch.cuda.synchronize()
    ro, rs = run_oracle(inp, H, W, 2)
    assert_parity(out.float().cpu().numpy(), ro, "out")
    assert_parity(st.cpu().numpy(), rs, "carried state")


def test_split_sequence_resume():
    """Two calls over the two halves of a grid (rows), carrying the state, equal one call."""
    B, heads, H, W = 1, 2, 16, 12
    inp = make_inputs(B, heads, H, W, 64, 64, seed=21)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    full, sfull = gla.gtr_gla_fwd(t["q"], t["k"], t["v"], t["g"], H, W, 0, final_state=True)
    half = H // 2 * W
    top = {n: x[:, :half].contiguous() for n, x in t.items()}
    bot = {n: x[:, half:].contiguous() for n, x in t.items()}
    o1, s1 = gla.gtr_gla_fwd(top["q"], top["k"], top["v"], top["g"], H // 2, W, 0,
                             final_state=True)
    o2, s2 = gla.gtr_gla_fwd(bot["q"], bot["k"], bot["v"], bot["g"], H - H // 2, W, 0,
                             init_state=s1, final_state=True)
    torch.cuda.synchronize()
    ro, rs = run_oracle(inp, H, W, 0)
    both = torch.cat([o1, o2], dim=1).float().cpu().numpy()
    assert_parity(both, ro, "split out")
    assert_parity(s2.cpu().numpy(), rs, "split state")
    assert_parity(full.float().cpu().numpy(), ro, "full out")


def test_empty_grid_copies_state():
    dev = torch.device("cuda", 0)
    z = torch.zeros((1, 0, 2, 64), dtype=torch.float16, device=dev)
    s0 = torch.randn((1, 2, 64, 64), device=dev)
    out, sf = gla.gtr_gla_fwd(z, z, z, z, 0, 7, 0, init_state=s0, final_state=True)
    torch.cuda.synchronize()
    assert out.shape == (1, 0, 2, 64)
    assert torch.equal(sf, s0)


def test_invalid_arguments_return_codes():
    dev = torch.device("cuda", 0)
    q = torch.zeros((1, 4, 1, 64), dtype=torch.float16, device=dev)
    o = torch.empty((1, 4, 1, 64), dtype=torch.float16, device=dev)
    p = q.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    # bad direction, bad chunk, unsupported dk, null pointer, misaligned, aliasing
    assert gla.gtr_gla_fwd_raw(p, p, p, p, 1, 1, 2, 2, 64, 64, 4, 64, 0, o.data_ptr(), 0, s) == \
        gla.GTR_ERR_INVALID_ARG
    assert gla.gtr_gla_fwd_raw(p, p, p, p, 1, 1, 2, 2, 64, 64, 0, 32, 0, o.data_ptr(), 0, s) == \
        gla.GTR_ERR_UNSUPPORTED
    assert gla.gtr_gla_fwd_raw(p, p, p, p, 1, 1, 2, 2, 96, 64, 0, 64, 0, o.data_ptr(), 0, s) == \
        gla.GTR_ERR_UNSUPPORTED
    assert gla.gtr_gla_fwd_raw(0, p, p, p, 1, 1, 2, 2, 64, 64, 0, 64, 0, o.data_ptr(), 0, s) == \
        gla.GTR_ERR_INVALID_ARG
    assert gla.gtr_gla_fwd_raw(p + 2, p, p, p, 1, 1, 2, 2, 64, 64, 0, 64, 0, o.data_ptr(), 0,
                               s) == gla.GTR_ERR_INVALID_ARG
    assert gla.gtr_gla_fwd_raw(p, p, p, p, 1, 1, 2, 2, 64, 64, 0, 64, 0, p, 0, s) == \
        gla.GTR_ERR_INVALID_ARG
    assert gla.device_status() == gla.GTR_OK


def test_large_sample_rows_match_oracle_subset():
    """Full-size 16.4K-token call; outputs of a few sequences checked against the oracle
    run on those sequences alone (sequences are independent)."""
    w = WORKLOADS["hires_b1h16_128x128"]
    inp = workload_inputs(w, 3, 7)
    out, sf = run_gpu(inp, w.H, w.W, 3)
    for h in (0, 9, 15):
        sub = {n: inp[n][:, :, h:h + 1].contiguous() for n in ("q", "k", "v", "g")}
        sub["s0"] = inp["s0"][:, h:h + 1].contiguous()
        ro, rs = run_oracle(sub, w.H, w.W, 3)
        assert_parity(out[:, :, h:h + 1], ro, f"head {h} out")
        assert_parity(sf[:, h:h + 1], rs, f"head {h} state")
