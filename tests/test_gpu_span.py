"""Span decomposition of the dk = 64 kernel vs the fp64 oracle (GPU only).

One sequence is cut into spans that run on different SMs from a zero state; each
later span looks back over its predecessors' aggregates and then adds the missing
initial-state term to its outputs: exactly by one extra MMA for the first chunks
of the span (kept in TMEM), by re-reading q, g and the stored output for the later
ones, or not at all when a bound shows the term is below 2^-16 of the chunk's
largest output.  The span count is forced with GTR_CLUSTER_SIZE so that every one
of those paths runs: near-1 retention makes the term large everywhere (re-reads),
strong forgetting makes it vanish (skips).
"""
import numpy as np
import pytest
import torch

from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import WORKLOADS, make_inputs, workload_inputs
from tests.gpu_common import assert_parity, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

AGG_FLOATS = 64 * 64 + 64   # per (sequence, span): state + decay product


def _z(mode):
    def z_of(shape):
        gen = torch.Generator().manual_seed(11)
        z = torch.randn(shape, generator=gen)
        if mode == "retain":      # a ~ 0.9998: the carried state barely decays
            return z + 6.0
        if mode == "forget":      # a ~ 0.8: the carried term vanishes within a chunk or two
            return z - 4.0
        if mode == "mixed":       # channels alternate between the two
            ch = torch.arange(shape[-1]).remainder(2).float()
            return z + 6.0 * ch - 4.0 * (1 - ch)
        return z
    return z_of


@pytest.mark.parametrize("spans", [2, 3, 4, 7, 13])
@pytest.mark.parametrize("mode", ["normal", "retain", "forget", "mixed"])
def test_forced_span_counts(monkeypatch, spans, mode):
    B, heads, H, W = 1, 4, 40, 40   # 25 chunks
    monkeypatch.setenv("GTR_CLUSTER_SIZE", str(spans))
    assert gla.plan(B, heads, H, W, 64, 64)[0] == spans
    inp = make_inputs(B, heads, H, W, 64, 64, seed=100 + spans, init_std=0.4,
                      z_override=_z(mode))
    for d in ((0, 1, 2, 3) if spans == 2 else (0, 3)):
        out, sf = run_gpu(inp, H, W, d)
        ro, rs = run_oracle(inp, H, W, d)
        assert_parity(out, ro, f"P={spans} {mode} dir {d} out")
        assert_parity(sf, rs, f"P={spans} {mode} dir {d} state")


@pytest.mark.parametrize("mode", ["normal", "retain"])
def test_long_spans_reread(monkeypatch, mode):
    """64 chunks in two spans of 32: 27 chunks of the second span take the re-read
    (or the skip) path."""
    B, heads, H, W = 1, 2, 64, 64
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "2")
    assert gla.plan(B, heads, H, W, 64, 64)[0] == 2
    inp = make_inputs(B, heads, H, W, 64, 64, seed=5, init_std=0.3, z_override=_z(mode))
    for d in (1, 2):
        out, sf = run_gpu(inp, H, W, d)
        ro, rs = run_oracle(inp, H, W, d)
        assert_parity(out, ro, f"{mode} dir {d} out")
        assert_parity(sf, rs, f"{mode} dir {d} state")


def test_ragged_last_span(monkeypatch):
    """Spans of 3 chunks over 25 chunks with a 1-chunk last span and a ragged tail."""
    B, heads, H, W = 2, 3, 39, 41    # 1599 tokens: 24 full chunks + 63
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "9")
    assert gla.plan(B, heads, H, W, 64, 64)[0] == 9
    inp = make_inputs(B, heads, H, W, 64, 64, seed=8, init_std=0.5, z_override=_z("mixed"))
    for d in range(4):
        out, sf = run_gpu(inp, H, W, d)
        ro, rs = run_oracle(inp, H, W, d)
        assert_parity(out, ro, f"dir {d} out")
        assert_parity(sf, rs, f"dir {d} state")


def test_span_groups_loop_over_sequences(monkeypatch):
    """100 sequences in two spans each: 74 span pairs, so CTAs loop over sequences."""
    B, heads, H, W = 5, 20, 16, 16
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "2")
    P, groups, _ = gla.plan(B, heads, H, W, 64, 64)
    assert P == 2 and groups < B * heads
    inp = make_inputs(B, heads, H, W, 64, 64, seed=13, init_std=0.2, z_override=_z("retain"))
    out, sf = run_gpu(inp, H, W, 2)
    ro, rs = run_oracle(inp, H, W, 2)
    assert_parity(out, ro, "out")
    assert_parity(sf, rs, "state")


def test_in_place_carry_with_spans(monkeypatch):
    B, heads, H, W = 1, 3, 24, 24
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "4")
    inp = make_inputs(B, heads, H, W, 64, 64, seed=31, init_std=0.3, z_override=_z("retain"))
    dev = torch.device("cuda", 0)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "g"))
    st = inp["s0"].to(dev).clone()
    out, _ = gla.gtr_gla_fwd(q, k, v, g, H, W, 1, init_state=st, final_state=st)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    ro, rs = run_oracle(inp, H, W, 1)
    assert_parity(out.float().cpu().numpy(), ro, "out")
    assert_parity(st.cpu().numpy(), rs, "carried state")


def _flags_clear(ws):
    """The workspace's publish flags (2 x 128 bytes per SM, rounded up to 256) are zero:
    every reader of a span's aggregate took itself off that span's flag."""
    sms = torch.cuda.get_device_properties(ws.device).multi_processor_count
    n = (2 * 128 * sms + 255) // 256 * 256
    return int(torch.count_nonzero(ws[:n]).item()) == 0


def test_caller_workspace_matches_default():
    w = WORKLOADS["gtr640_b1h16_40x40"]
    dev = torch.device("cuda", 0)
    P, _, _ = gla.plan(w.B, w.heads, w.H, w.W, w.dk, w.dv)
    nbytes = gla.workspace_bytes(w.B, w.heads, w.H, w.W, w.dk, w.dv)
    assert P > 1 and nbytes > 0
    ws = gla.new_workspace(nbytes, dev)
    for call, d in enumerate((0, 3, 1)):
        inp = workload_inputs(w, d, call + 40)
        t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
        s0 = inp["s0"].to(dev) if inp["s0"] is not None else None
        o1, s1 = gla.gtr_gla_fwd_ws(t["q"], t["k"], t["v"], t["g"], w.H, w.W, d, ws,
                                    init_state=s0, final_state=True)
        o2, s2 = gla.gtr_gla_fwd(t["q"], t["k"], t["v"], t["g"], w.H, w.W, d, init_state=s0,
                                 final_state=True)
        torch.cuda.synchronize()
        assert gla.device_status() == gla.GTR_OK
        assert torch.equal(o1, o2) and torch.equal(s1, s2)
        assert _flags_clear(ws)
        ro, rs = run_oracle(inp, w.H, w.W, d)
        assert_parity(o1.float().cpu().numpy(), ro, f"call {call} out")
        assert_parity(s1.cpu().numpy(), rs, f"call {call} state")


def test_workspace_shared_across_shapes(monkeypatch):
    """One workspace (and the library's own) reused by calls whose span plans differ:
    aggregates of one plan must never be read as another plan's publish flags."""
    dev = torch.device("cuda", 0)
    shapes = [(1, 4, 40, 40, 2, "retain"), (1, 4, 40, 40, 3, "normal"), (2, 3, 24, 32, 4, "retain"),
              (1, 4, 40, 40, 2, "normal"), (1, 2, 33, 35, 7, "mixed")]
    need = 0
    for B, heads, H, W, P, _ in shapes:
        monkeypatch.setenv("GTR_CLUSTER_SIZE", str(P))
        need = max(need, gla.workspace_bytes(B, heads, H, W, 64, 64))
    ws = gla.new_workspace(need, dev)
    for rep in range(2):
        for i, (B, heads, H, W, P, mode) in enumerate(shapes):
            monkeypatch.setenv("GTR_CLUSTER_SIZE", str(P))
            inp = make_inputs(B, heads, H, W, 64, 64, seed=300 + 10 * i + rep, init_std=0.3,
                              z_override=_z(mode))
            t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
            s0 = inp["s0"].to(dev)
            d = (i + rep) % 4
            o1, s1 = gla.gtr_gla_fwd_ws(t["q"], t["k"], t["v"], t["g"], H, W, d, ws,
                                        init_state=s0, final_state=True)
            o2, s2 = gla.gtr_gla_fwd(t["q"], t["k"], t["v"], t["g"], H, W, d, init_state=s0,
                                     final_state=True)
            torch.cuda.synchronize()
            assert gla.device_status() == gla.GTR_OK
            assert _flags_clear(ws)
            ro, rs = run_oracle(inp, H, W, d)
            for what, o, st in (("caller ws", o1, s1), ("library ws", o2, s2)):
                assert_parity(o.float().cpu().numpy(), ro, f"{what} shape {i} rep {rep} out")
                assert_parity(st.cpu().numpy(), rs, f"{what} shape {i} rep {rep} state")


def test_workspace_argument_checks():
    w = WORKLOADS["gtr640_b1h16_40x40"]
    dev = torch.device("cuda", 0)
    nbytes = gla.workspace_bytes(w.B, w.heads, w.H, w.W, w.dk, w.dv)
    inp = workload_inputs(w, 0, 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    args = (t["q"], t["k"], t["v"], t["g"], w.H, w.W, 0)
    for bad in (None, gla.new_workspace(nbytes - 256, dev), gla.new_workspace(nbytes + 512, dev)[16:]):
        with pytest.raises(gla.GTRError) as e:
            gla.gtr_gla_fwd_ws(*args, bad)
        assert e.value.status == gla.GTR_ERR_INVALID_ARG
    # shapes with many sequences need none
    big = WORKLOADS["b8h16_48x48_stack12"]
    assert gla.workspace_bytes(big.B, big.heads, big.H, big.W, big.dk, big.dv) == 0
    assert gla.workspace_bytes(1, 1, 4, 4, 64, 64, chunk=32) == 0
    assert gla.device_status() == gla.GTR_OK
