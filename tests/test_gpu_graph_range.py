"""The timed configuration and the numeric range, against the fp64 oracle (GPU only).

* bench.py times a CUDA graph of back-to-back calls: eight rotating input sets x four
  scan directions, programmatic dependent launch (each call's set-up overlapping the
  previous call's tail) and the library's shared workspace.  The graph is replayed
  twice here, exactly as the bench replays it, and every output and final state of
  the last replay is compared with the oracle.
* Large-magnitude inputs: keys of magnitude above 100 take the sub-block path by
  magnitude (not by decay) and must still match the oracle; inputs whose running
  state or scores cannot be represented in fp16 must be reported as GTR_ERR_RANGE,
  never returned silently as wrong numbers.
"""
import numpy as np
import pytest
import torch

import bench
from recurrent_vision_backbone_b200 import gla
from recurrent_vision_backbone_b200.inputs import DIR_NAMES, WORKLOADS, make_inputs
from tests.gpu_common import assert_parity, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["gtr640_b1h16_40x40", "pr1_b1h4_20x20"])
def test_bench_graph_replay_matches_oracle(name):
    w = WORKLOADS[name]
    dev = torch.device("cuda", 0)
    wl = bench.Workload(w, 0, dev, n_sets=8)
    stream = torch.cuda.Stream(device=dev)
    wl.capture(stream, 8)
    with torch.cuda.stream(stream):
        wl.replay(16)   # two rotations back to back: every call is preceded by another
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_OK
    for s, calls in enumerate(wl.sets):
        for d, inp, out, sf in calls:
            host = {n: (None if t is None else t.cpu()) for n, t in inp.items()}
            ro, rs = run_oracle(host, w.H, w.W, d)
            what = f"set {s} {DIR_NAMES[d]}"
            assert_parity(out.float().cpu().numpy(), ro, what + " out")
            if sf is not None:
                assert_parity(sf.cpu().numpy(), rs, what + " final state")


def _scaled_inputs(B, heads, H, W, seed, kscale, init_std=0.3):
    inp = make_inputs(B, heads, H, W, 64, 64, seed=seed, init_std=init_std)
    inp["k"] = (inp["k"].float() * kscale).half()
    return inp


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_large_keys_take_the_sub_block_path_and_match(direction):
    """|k| up to ~600 (> 100: the fast path's key bound) with the pages' gates."""
    B, heads, H, W = 1, 4, 24, 40
    inp = _scaled_inputs(B, heads, H, W, seed=41 + direction, kscale=150.0)
    assert float(inp["k"].float().abs().max()) > 100.0
    out, sf = run_gpu(inp, H, W, direction)
    ro, rs = run_oracle(inp, H, W, direction)
    assert_parity(out, ro, "out")
    assert_parity(sf, rs, "final state")


def test_large_keys_with_spans_match(monkeypatch):
    """The same magnitudes with the sequence split into spans (look-back and corrections
    see large aggregates)."""
    B, heads, H, W = 1, 4, 40, 40
    monkeypatch.setenv("GTR_CLUSTER_SIZE", "5")
    inp = _scaled_inputs(B, heads, H, W, seed=47, kscale=120.0)
    for d in (1, 2):
        out, sf = run_gpu(inp, H, W, d)
        ro, rs = run_oracle(inp, H, W, d)
        assert_parity(out, ro, f"dir {d} out")
        assert_parity(sf, rs, f"dir {d} final state")


def _positive_retain_inputs(H, W, mag):
    """All-positive keys and values with no decay: the state grows linearly with the
    number of tokens (mag^2 per token and entry)."""
    B, heads = 1, 2
    N = H * W
    q = torch.full((B, N, heads, 64), 2.0 ** -7, dtype=torch.float16)   # outputs = t * mag^2 / 2
    k = torch.full((B, N, heads, 64), mag, dtype=torch.float16)
    v = torch.full((B, N, heads, 64), mag, dtype=torch.float16)
    g = torch.zeros((B, N, heads, 64), dtype=torch.float16)
    return dict(q=q, k=k, v=v, g=g, s0=None)


def test_state_beyond_fp16_is_reported():
    """16384 tokens of k = v = 3 without decay: the state reaches 147456 > 65504."""
    H = W = 128
    inp = _positive_retain_inputs(H, W, 3.0)
    dev = torch.device("cuda", 0)
    t = {n: inp[n].to(dev) for n in ("q", "k", "v", "g")}
    gla.gtr_gla_fwd(t["q"], t["k"], t["v"], t["g"], H, W, 0, final_state=True)
    torch.cuda.synchronize()
    assert gla.device_status() == gla.GTR_ERR_RANGE
    assert gla.device_status() == gla.GTR_OK   # read and cleared


def test_state_inside_fp16_is_exact():
    """The same construction with k = v = 1: the state ends at 16384 and the outputs at
    8192 (inside fp16)."""
    H = W = 128
    inp = _positive_retain_inputs(H, W, 1.0)
    out, sf = run_gpu(inp, H, W, 2)
    ro, rs = run_oracle(inp, H, W, 2)
    assert_parity(out, ro, "out")
    assert_parity(sf, rs, "final state")
