"""Throughput benchmark of the GTR token-mixer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

One step = one layer call per scan direction (L->R, R->L, T->B, B->T) of the
1.6K-token workload (B=1, 16 heads, 40x40 patch grid, dk=dv=64, fp16, chunk 64),
each call on its own freshly drawn inputs.  The metric is spatial tokens per
second (B*N per call, all heads included) over the whole job.  The same line
also reports the 16.4K-token workload (B=1, 16 heads, 128x128) measured the
same way.

Inputs live in HBM before timing starts and rotate over enough distinct sets
that their footprint is several times the 126 MB L2, so no call reads inputs
the previous ones left in L2.  The timed steps are replayed from a CUDA graph
(the launches would otherwise be host-bound), bracketed by a barrier and a
device synchronise, timed with CUDA events, max over ranks.  Under torchrun each
rank runs its own independent batch (weak scaling, no collective in the data
path).  ``--impl reference`` times the fp64 CPU oracle on this host's cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from recurrent_vision_backbone_b200.inputs import DIR_NAMES, TAU, WORKLOADS, make_inputs  # noqa: E402

METRIC = "GLA fwd tokens/s at 1.6K & 16.4K tokens (FP16, C=64); % of roofline"
PRIMARY = "gtr640_b1h16_40x40"
SECONDARY = "hires_b1h16_128x128"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
DIRS = (0, 1, 2, 3)


# ------------------------------------------------------------------ accounting
def bytes_alg(w) -> int:
    """Algorithmic HBM bytes of one call: read q, k, g, v and write o once (fp16),
    plus the fp32 initial and final states where the workload has them."""
    th = w.B * w.N * w.heads
    b = th * 2 * (3 * w.dk + 2 * w.dv)
    per_state = w.B * w.heads * w.dk * w.dv * 4
    if w.init_std:
        b += per_state
    if w.final_state:
        b += per_state
    return b


def flops_alg(w, chunk=64) -> int:
    """Algorithmic FLOPs of one call: causal intra-chunk term, inter-chunk term and
    state update (per token-head (C+1)(dk+dv) + 4 dk dv)."""
    th = w.B * w.N * w.heads
    return th * ((chunk + 1) * (w.dk + w.dv) + 4 * w.dk * w.dv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_tokens(src: str) -> str:
    """C++ source without comments, whitespace runs collapsed (string and character
    literals kept verbatim): edits to comments or layout leave it unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


KERNEL_FILES = {"gla_fwd_span_kernel": "gla_fwd_span.cuh", "gla_fwd_pipe_kernel": "gla_fwd_pipe.cuh",
                "swiglu_gate_kernel": "swiglu_gate.cuh", "gla_bwd_grad_kernel": "gla_bwd.cuh"}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code a kernel is built from (comments and layout excluded): its own
    file, the PTX wrappers and the shared device part of gtr_gla.cu (up to its host
    section), recorded next to the ncu counters in profiles/ so that a stale capture
    is not reported."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "recurrent_vision_backbone_b200", "csrc")
    for name in (KERNEL_FILES[kernel], "sm100_ptx.cuh", "gtr_gla.cu"):
        with open(os.path.join(csrc, name), encoding="utf-8") as fh:
            text = fh.read()
        if name == "gtr_gla.cu":
            text = text[:text.index("// ------------------------------------------------------------------ host")]
        h.update(_code_tokens(text).encode())
    return h.hexdigest()[:12]


def kernel_for(w, gate_z=False) -> str:
    """The kernel a call of workload w launches (a dk = 128 call: twice); the same for
    the gate-from-z entry (an instance that reads z)."""
    if os.environ.get("GTR_KERNEL") == "pipe":
        return "gla_fwd_pipe_kernel"
    return "gla_fwd_span_kernel"


def launches_per_call(w) -> int:
    """dk = 128 runs as two launches over the two 64-channel key halves."""
    return 2 if w.dk == 128 else 1


def recorded_profile(workload_name: str, key: str = "traffic_bytes_per_call"):
    """A number from the committed ncu summary of the workload's kernel (DRAM bytes
    per call, warp instructions per chunk), if it was taken on the current kernel
    source; else None.  (A name ending in "+z": the gate-from-z entry.)"""
    gate_z = workload_name.endswith("+z")
    kernel = kernel_for(WORKLOADS[workload_name[:-2] if gate_z else workload_name], gate_z)
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload_name}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"kernel_source_sha1:\s*([0-9a-f]+)", text)
    m_v = re.search(key + r":\s*([0-9.]+)", text)
    if not m_sha or not m_v or m_sha.group(1) != kernel_source_hash(kernel):
        return None
    return float(m_v.group(1)) if "." in m_v.group(1) else int(m_v.group(1))


def recorded_traffic(workload_name: str):
    return recorded_profile(workload_name, "traffic_bytes_per_call")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path=None):
        """Samples the GPU's clocks every 100 ms while the timed region runs; the raw
        samples go to `path` (a CSV) if given, else to a temporary file."""
        self.gpu = gpu_index
        self.proc = None
        self.temporary = path is None
        if path is None:
            fd, path = tempfile.mkstemp(prefix=f"clocks_gpu{gpu_index}_", suffix=".csv")
            os.close(fd)
        self.path = path

    def start(self):
        try:
            if os.path.dirname(self.path):
                os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            if self.temporary and os.path.exists(self.path):
                os.unlink(self.path)
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        if self.temporary:
            os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ ranks
def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's inputs: every rank draws its own independent batch (weak scaling)."""
    return int(base_seed) + 7919 * int(rank)


def shard_sequences(n_seq: int, world: int, rank: int) -> range:
    """Contiguous slice of the (batch, head) sequences a rank owns when one batch is split
    across ranks; sequences are independent, so no collective is needed on the data path."""
    lo = n_seq * rank // world
    hi = n_seq * (rank + 1) // world
    return range(lo, hi)


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank measurement over all ranks (timings are reported as the max)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ GPU arm
class Workload:
    """Rotating device-resident input sets for one workload and the graph that
    replays `group` steps of 4 direction calls over them."""

    def __init__(self, w, rank, device, n_sets=None, gate_z=False):
        from recurrent_vision_backbone_b200 import gla
        self.gla = gla
        self.w = w
        self.gate_z = gate_z   # gtr_gla_fwd_z: the gate's pre-activation z in place of g
        per_call = bytes_alg(w)
        if n_sets is None:
            n_sets = max(4, -(-4 * L2_BYTES // (per_call * len(w.call_directions()))))
        self.n_sets = int(n_sets)
        self.sets = []
        for s in range(self.n_sets):
            calls = []
            for c, d in enumerate(w.call_directions()):
                inp = make_inputs(w.B, w.heads, w.H, w.W, w.dk, w.dv,
                                  seed=rank_seed(w.seed(d, 100 + 16 * s + c), rank),
                                  init_std=w.init_std, z_mean_per_head=w.z_mean_per_head,
                                  device=device, with_z=gate_z)
                if gate_z:
                    del inp["g"]
                out = torch.empty((w.B, w.N, w.heads, w.dv), dtype=torch.float16, device=device)
                sf = (torch.empty((w.B, w.heads, w.dk, w.dv), dtype=torch.float32, device=device)
                      if w.final_state else None)
                calls.append((d, inp, out, sf))
            self.sets.append(calls)
        self.graph = None

    def launch_step(self, s, stream):
        for d, inp, out, sf in self.sets[s % self.n_sets]:
            if self.gate_z:
                self.gla.gtr_gla_fwd_z(inp["q"], inp["k"], inp["v"], inp["z"], TAU, self.w.H, self.w.W, d,
                                       init_state=inp["s0"], out=out, final_state=sf, stream=stream)
            else:
                self.gla.gtr_gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"], self.w.H, self.w.W, d,
                                     init_state=inp["s0"], out=out, final_state=sf, stream=stream)

    def capture(self, stream, steps):
        """Graphs replaying the rotating sets: `graph` holds one step per set; a graph of
        the first r sets serves any step count with remainder r (the one of `steps` is
        recorded here, others when first replayed, outside any timed region)."""
        with torch.cuda.stream(stream):   # warm the launch path once outside capture
            self.launch_step(0, stream)
        stream.synchronize()
        self.stream = stream
        self.parts = {}
        self.graph = self._graph_of(self.n_sets)
        self._part(steps % self.n_sets)
        return self.n_sets

    def _graph_of(self, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for s in range(n):
                self.launch_step(s, torch.cuda.current_stream())
        return g

    def _part(self, r):
        if r and r not in self.parts:
            self.parts[r] = self._graph_of(r)
        return self.parts.get(r)

    def replay(self, steps):
        """Replays exactly `steps` steps (whole rotations, then the remainder)."""
        part = self._part(steps % self.n_sets)
        for _ in range(steps // self.n_sets):
            self.graph.replay()
        if part is not None:
            part.replay()

    def calls_per_step(self):
        return len(self.w.call_directions())

    def tokens_per_step(self):
        return self.calls_per_step() * self.w.B * self.w.N


def timed_replays(wl, steps, stream, world):
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):   # replay on the stream the events are recorded on
        start.record(stream)
        wl.replay(steps)
        end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(start.elapsed_time(end), world, "cuda")


def measure(wl, steps, warmup, stream, world, clocks=None, clock_window_s=1.0):
    """W warm-up steps, then exactly `steps` timed steps.  With a clock sampler, the
    samples cover a window of at least `clock_window_s` of the same replays that ends
    with the timed region (a timed region of a few ms holds no 100 ms sample)."""
    per_replay = wl.capture(stream, steps)
    with torch.cuda.stream(stream):
        wl.replay(max(warmup, 1))
    torch.cuda.synchronize()
    assert wl.gla.device_status() == wl.gla.GTR_OK
    clk = None
    if clocks is not None:
        # size the untimed lead-in from one timed rotation
        t_rot = timed_replays(wl, per_replay, stream, world) * 1e-3
        lead = max(0, int(clock_window_s / max(t_rot, 1e-6)) + 1)
        clocks.start()
        with torch.cuda.stream(stream):
            for _ in range(lead):
                wl.graph.replay()
    ms = timed_replays(wl, steps, stream, world)
    if clocks is not None:
        clk = clocks.stop()
    assert wl.gla.device_status() == wl.gla.GTR_OK
    return ms, steps, clk


def roofline(w, ms_per_call, workload_name, gate_z=False):
    peak, which = measured_peaks()
    b = bytes_alg(w)
    achieved = b / (ms_per_call * 1e-3) / 1e9
    return {"kernel": kernel_for(w, gate_z), "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": recorded_traffic(workload_name),
            "peak_source": which, "bytes_alg_per_call": b, "flops_alg_per_call": flops_alg(w),
            "launches_per_call": launches_per_call(w),
            # the issue bound: warp instructions per 64-token chunk of one sequence
            "inst_per_chunk": recorded_profile(workload_name, "inst_per_chunk")}


# ------------------------------------------------------------------ Spatial SwiGLU
def swiglu_bytes_alg(w) -> int:
    """Read U and G, write h (fp16), plus the fp32 kernel and bias."""
    return 6 * w.B * w.N * w.C + 40 * w.C


class SwigluBench:
    """Rotating device-resident input sets of one Spatial SwiGLU workload, one
    gtr_spatial_swiglu_gate call per step, replayed from CUDA graphs (the interface
    of Workload, for measure())."""

    def __init__(self, w, device, n_sets=None):
        from recurrent_vision_backbone_b200 import gla
        from recurrent_vision_backbone_b200.inputs import make_swiglu_inputs
        self.gla = gla
        self.w = w
        if n_sets is None:
            n_sets = max(4, -(-4 * L2_BYTES // swiglu_bytes_alg(w)))
        self.n_sets = int(n_sets)
        self.sets = []
        for s in range(self.n_sets):
            inp = make_swiglu_inputs(w.B, w.H, w.W, w.C, seed=5000 + s, device=device)
            self.sets.append((inp, torch.empty_like(inp["G"])))

    def launch_step(self, s, stream):
        inp, out = self.sets[s % self.n_sets]
        self.gla.gtr_spatial_swiglu_gate(inp["G"], inp["U"], inp["w"], inp["bias"], out=out, stream=stream)

    capture = Workload.capture
    _graph_of = Workload._graph_of
    _part = Workload._part
    replay = Workload.replay

    def calls_per_step(self):
        return 1


def run_swiglu(name, steps, warmup, stream, world, device, sets, local):
    from recurrent_vision_backbone_b200.inputs import SWIGLU_WORKLOADS
    w = SWIGLU_WORKLOADS[name]
    sb = SwigluBench(w, device, n_sets=sets)
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    ms, n_steps, clk = measure(sb, steps, warmup, stream, world, clocks)
    peak, which = measured_peaks()
    b = swiglu_bytes_alg(w)
    achieved = b / (ms / n_steps * 1e-3) / 1e9
    res = {"workload": name, "tokens_per_call": w.B * w.N, "channels": w.C,
           "value": round(world * w.B * w.N * n_steps / (ms * 1e-3), 1), "unit": "tokens/s",
           "steps": n_steps, "us_per_call": round(ms * 1e3 / n_steps, 3),
           "roofline": {"kernel": "swiglu_gate_kernel", "bound": "hbm", "achieved": round(achieved, 1),
                        "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                        "traffic": recorded_traffic_swiglu(name), "peak_source": which,
                        "bytes_alg_per_call": b, "launches_per_call": 1},
           "gpu_launches": n_steps, "clocks": clk,
           "l2": f"inputs rotate over {sb.n_sets} sets ({sb.n_sets * b / 2**20:.0f} MiB > 3x L2)"}
    del sb
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ backward
BWD_WORKLOADS = ("gtr640_b1h16_40x40", "hires_b1h16_128x128")


def bwd_bytes_alg(w) -> int:
    """Algorithmic HBM bytes of one backward call: read q, k, g, v and d_out (fp16),
    write grad_q, grad_k, grad_g and grad_v (fp32), plus the fp32 states it reads
    (init_state, d_final_state) and writes (grad_init_state)."""
    th = w.B * w.N * w.heads
    b = th * (2 * (3 * w.dk + 2 * w.dv) + 4 * (3 * w.dk + w.dv))
    per_state = w.B * w.heads * w.dk * w.dv * 4
    return b + per_state * (int(bool(w.init_std)) + 2 * int(bool(w.final_state)))


class BwdBench:
    """Rotating device-resident sets of one workload's backward calls (one per direction
    per step, each with its own inputs, upstream gradients and gradient outputs; one
    workspace, the calls being stream-ordered), replayed from CUDA graphs."""

    def __init__(self, w, device, n_sets=None, rank=0):
        from recurrent_vision_backbone_b200 import gla
        from recurrent_vision_backbone_b200.inputs import make_upstream
        self.gla = gla
        self.w = w
        per_step = bwd_bytes_alg(w) * len(w.directions)
        if n_sets is None:
            n_sets = max(2, -(-4 * L2_BYTES // per_step))
        self.n_sets = int(n_sets)
        self.ws = gla.new_workspace(gla.bwd_workspace_bytes(w.B, w.heads, w.H, w.W, w.dk, w.dv), device)
        f32 = dict(dtype=torch.float32, device=device)
        self.sets = []
        for s in range(self.n_sets):
            calls = []
            for d in w.directions:
                seed = rank_seed(w.seed(d, 300 + s), rank)   # each rank its own batch
                inp = make_inputs(w.B, w.heads, w.H, w.W, w.dk, w.dv, seed=seed, init_std=w.init_std,
                                  z_mean_per_head=w.z_mean_per_head, device=device)
                d_out, dsf = make_upstream(w.B, w.heads, w.H, w.W, w.dk, w.dv, seed, with_dsf=w.final_state,
                                           device=device)
                grads = (torch.empty((w.B, w.N, w.heads, w.dk), **f32), torch.empty((w.B, w.N, w.heads, w.dk), **f32),
                         torch.empty((w.B, w.N, w.heads, w.dv), **f32), torch.empty((w.B, w.N, w.heads, w.dk), **f32),
                         torch.empty((w.B, w.heads, w.dk, w.dv), **f32) if w.final_state else None)
                calls.append((d, inp, d_out, dsf, grads))
            self.sets.append(calls)

    def launch_step(self, s, stream):
        for d, inp, d_out, dsf, grads in self.sets[s % self.n_sets]:
            self.gla.gtr_gla_bwd(inp["q"], inp["k"], inp["v"], inp["g"], d_out, self.w.H, self.w.W, d,
                                 init_state=inp["s0"], d_final_state=dsf, workspace=self.ws, grads=grads,
                                 stream=stream)

    capture = Workload.capture
    _graph_of = Workload._graph_of
    _part = Workload._part
    replay = Workload.replay

    def calls_per_step(self):
        return len(self.w.directions)


BWD_KERNELS_PER_CALL = 4   # chunk locals, state scans, chunk gradients, dg offsets


def run_bwd(name, steps, warmup, stream, world, device, sets, local, rank=0):
    w = WORKLOADS[name]
    bb = BwdBench(w, device, n_sets=sets, rank=rank)
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    ms, n_steps, clk = measure(bb, steps, warmup, stream, world, clocks)
    peak, which = measured_peaks()
    calls = n_steps * bb.calls_per_step()
    b = bwd_bytes_alg(w)
    achieved = b / (ms / calls * 1e-3) / 1e9
    res = {"workload": name + "+bwd", "entry": "gtr_gla_bwd", "tokens_per_call": w.B * w.N,
           "value": round(world * w.B * w.N * calls / (ms * 1e-3), 1), "unit": "tokens/s",
           "steps": n_steps, "us_per_call": round(ms * 1e3 / calls, 3),
           "roofline": {"kernel": "gla_bwd_*", "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                        "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                        "peak_source": which, "bytes_alg_per_call": b,
                        "launches_per_call": BWD_KERNELS_PER_CALL * (w.dk // 64)},
           "gpu_launches": calls * BWD_KERNELS_PER_CALL * (w.dk // 64), "clocks": clk,
           "l2": f"inputs rotate over {bb.n_sets} sets ({bb.n_sets * b * bb.calls_per_step() / 2**20:.0f} MiB > 3x L2)"}
    del bb
    torch.cuda.empty_cache()
    return res


def recorded_traffic_swiglu(name: str):
    path = os.path.join(ROOT, "profiles", f"swiglu_gate_kernel_{name}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"kernel_source_sha1:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"traffic_bytes_per_call:\s*([0-9]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != kernel_source_hash("swiglu_gate_kernel"):
        return None
    return int(m_tr.group(1))


def call_inputs(w, d, seed, heads=None, device="cpu"):
    """Inputs of one call of workload w (optionally only its first `heads` heads)."""
    h = w.heads if heads is None else heads
    zm = None if w.z_mean_per_head is None else tuple(w.z_mean_per_head[:h])
    return make_inputs(w.B, h, w.H, w.W, w.dk, w.dv, seed=seed, init_std=w.init_std,
                       z_mean_per_head=zm, device=device)


def e2e_measure(w, steps, device, rank):
    """Tokens/s through the public call with host buffers: every step copies that
    step's inputs from pinned host memory and reads its outputs back.  Uploads,
    calls and read-backs run on three streams (PCIe carries both directions at
    once), with two sets of device buffers so that step s+1's uploads overlap step
    s's read-backs; events order every reuse of a buffer."""
    from recurrent_vision_backbone_b200 import gla
    calls = []
    for c, d in enumerate(w.call_directions()):
        inp = call_inputs(w, d, rank_seed(w.seed(d, 500 + c), rank))
        hp = {n: t.pin_memory() for n, t in inp.items() if t is not None}
        sets = []
        for _ in range(2):
            dv = {n: torch.empty_like(t, device=device) for n, t in hp.items()}
            out = torch.empty((w.B, w.N, w.heads, w.dv), dtype=torch.float16, device=device)
            sf = (torch.empty((w.B, w.heads, w.dk, w.dv), dtype=torch.float32, device=device)
                  if w.final_state else None)
            ev = {k: torch.cuda.Event() for k in ("up", "done", "down")}
            sets.append((dv, out, sf, ev))
        h_out = torch.empty((w.B, w.N, w.heads, w.dv), dtype=torch.float16).pin_memory()
        h_sf = (torch.empty((w.B, w.heads, w.dk, w.dv), dtype=torch.float32).pin_memory()
                if w.final_state else None)
        calls.append((d, hp, sets, h_out, h_sf))
    s_up, s_call, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    h2d = sum(t.numel() * t.element_size() for c in calls for t in c[1].values())
    d2h = sum(c[3].numel() * c[3].element_size() + (0 if c[4] is None else
                                                   c[4].numel() * c[4].element_size())
              for c in calls)
    used = set()

    def one_step(step):
        par = step & 1
        for ci, (d, hp, sets, h_out, h_sf) in enumerate(calls):
            dv, out, sf, ev = sets[par]
            first = (ci, par) not in used
            used.add((ci, par))
            with torch.cuda.stream(s_up):
                if not first:
                    s_up.wait_event(ev["done"])      # the call two steps back read dv
                for n, t in hp.items():
                    dv[n].copy_(t, non_blocking=True)
                ev["up"].record(s_up)
            with torch.cuda.stream(s_call):
                s_call.wait_event(ev["up"])
                if not first:
                    s_call.wait_event(ev["down"])    # out / sf of two steps back read back
                gla.gtr_gla_fwd(dv["q"], dv["k"], dv["v"], dv["g"], w.H, w.W, d,
                                init_state=dv.get("s0"), out=out, final_state=sf, stream=s_call)
                ev["done"].record(s_call)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev["done"])
                h_out.copy_(out, non_blocking=True)
                if sf is not None:
                    h_sf.copy_(sf, non_blocking=True)
                ev["down"].record(s_down)

    for i in range(3):
        one_step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_up)
    s_call.wait_event(start)
    s_down.wait_event(start)
    for i in range(steps):
        one_step(3 + i)
    s_down.wait_event(calls[-1][2][(3 + steps - 1) & 1][3]["down"])
    s_down.wait_stream(s_up)
    s_down.wait_stream(s_call)
    end.record(s_down)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    return ms, steps, h2d, d2h


def config_of(w, world, l2_note, timing, gate_z=False):
    """The line's `config` (the same keys in both arms)."""
    return {"workload": w.name, "entry": "gtr_gla_fwd_z" if gate_z else "gtr_gla_fwd",
            "B": w.B, "heads": w.heads, "grid": [w.H, w.W],
            "tokens_per_call": w.B * w.N, "dk": w.dk, "dv": w.dv, "chunk": 64,
            "calls_per_step": len(w.call_directions()),
            "directions": ",".join(DIR_NAMES[d] for d in w.call_directions()),
            "l2": l2_note, "timing": timing,
            "parallelism": f"dp{world} (independent batches)"}


def run_workload(name, steps, warmup, stream, world, rank, device, sets, sample_clocks, local,
                 clocks_csv=None, gate_z=False):
    """Times `steps` steps of one workload; returns its numbers and its config.  gate_z:
    through gtr_gla_fwd_z (the gate's pre-activation z read in place of g: the same
    bytes, the gate formed in the kernel)."""
    w = WORKLOADS[name]
    wl = Workload(w, rank, device, n_sets=sets, gate_z=gate_z)
    clocks = None
    if sample_clocks:
        clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                              else local, clocks_csv)
    ms, n_steps, clk = measure(wl, steps, warmup, stream, world, clocks)
    calls = n_steps * wl.calls_per_step()
    res = {"workload": name + ("+z" if gate_z else ""), "tokens_per_call": w.B * w.N,
           "value": round(world * wl.tokens_per_step() * n_steps / (ms * 1e-3), 1),
           "unit": "tokens/s", "steps": n_steps, "ms_per_step": round(ms / n_steps, 6),
           "us_per_call": round(ms * 1e3 / calls, 3),
           # a call's bytes over a call's time (a dk = 128 call: both launches)
           "roofline": roofline(w, ms / calls, name + ("+z" if gate_z else ""), gate_z), "gpu_launches": calls * launches_per_call(w),
           "clocks": clk}
    l2 = (f"inputs rotate over {wl.n_sets} sets of {wl.calls_per_step()} calls "
          f"({wl.n_sets * wl.calls_per_step() * bytes_alg(w) / 2**20:.0f} MiB > 3x L2)")
    cfg = config_of(w, world, l2, "CUDA graph replay (exactly `steps` steps), CUDA events, "
                                  "max over ranks; clocks sampled over >= 1 s of the same "
                                  "replays ending with the timed region", gate_z)
    del wl
    torch.cuda.empty_cache()
    return res, cfg


# (workload, through the gate-from-z entry point)
SECONDARIES = (("hires_b1h16_128x128", False), ("b8h16_48x48_stack12", False),
               ("stress_b4h12_37x53_dk128", False), ("gtr640_b1h16_40x40", True),
               ("hires_b1h16_128x128", True))


def gpu_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", init_method="env://", timeout=timedelta(seconds=120),
                                device_id=device)
    from recurrent_vision_backbone_b200 import gla
    gla.load()
    stream = torch.cuda.Stream(device=device)
    primary = args.workload
    w1 = WORKLOADS[primary]
    res, cfg = run_workload(primary, args.steps, args.warmup, stream, world, rank, device,
                            args.sets, True, local, args.clocks_csv, gate_z=args.gate_z)
    line = {
        "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": res["steps"], "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic", "config": cfg, "roofline": res["roofline"],
        "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
        "us_per_call": res["us_per_call"],
    }
    if not args.no_secondary:
        line["secondary"] = []
        for name, gz in SECONDARIES:
            if name == primary and not gz:
                continue
            r2, _ = run_workload(name, max(8, args.steps // 16), max(3, args.warmup // 16), stream,
                                 world, rank, device, args.sets, True, local, gate_z=gz)
            line["secondary"].append(r2)
        from recurrent_vision_backbone_b200.inputs import SWIGLU_WORKLOADS
        for name in SWIGLU_WORKLOADS:   # the Spatial SwiGLU gated value branch
            line["secondary"].append(run_swiglu(name, max(8, args.steps // 16), max(3, args.warmup // 16),
                                                stream, world, device, None, local))
        for name in BWD_WORKLOADS:   # the backward pass
            line["secondary"].append(run_bwd(name, max(8, min(200, args.steps // 16)), 3, stream, world,
                                             device, None, local, rank=rank))
    # end to end through the public call with host buffers
    e_steps = max(3, min(args.steps, args.e2e_steps))
    ems, en, h2d, d2h = e2e_measure(w1, e_steps, device, rank)
    ems = max_over_ranks(ems, world, "cuda")
    wl_calls = len(w1.call_directions())
    line["e2e"] = {"value": round(world * wl_calls * w1.B * w1.N * en / (ems * 1e-3), 1),
                   "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "steps": en}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w1, budget_s=args.cpu_seconds)
    else:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ CPU arm
def cpu_baseline(w, budget_s=15.0):
    """The oracle as it stands, on this host's cores, on whole steps of the workload
    until the oracle time reaches the budget."""
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    tok, spent, steps = 0, 0.0, 0
    while spent < budget_s and steps < 1000:
        for c, d in enumerate(w.call_directions()):
            f = {n: t.float().numpy() for n, t in call_inputs(w, d, w.seed(d, 900 + c)).items()
                 if t is not None}
            t1 = time.perf_counter()
            oracle.gla_forward(f["q"], f["k"], f["v"], f["g"], w.H, w.W, d, f.get("s0"))
            spent += time.perf_counter() - t1
            tok += w.B * w.N
        steps += 1
    ncalls = steps * len(w.call_directions())
    return {"value": round(tok / spent, 1), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{steps} full steps ({ncalls} calls) of {w.name}, fp64 token-by-token, "
                      f"OpenMP over the {w.B * w.heads} sequences; oracle time only "
                      f"({spent:.1f} s)"}


def reference_arm(args):
    """The reference arm: the fp64 oracle on this host's cores, on a per-step sample of
    the workload's heads sized so that warmup + steps end within about two minutes."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    w = WORKLOADS[args.workload]
    dirs = w.call_directions()
    f = {n: t.float().numpy() for n, t in call_inputs(w, dirs[0], 1, heads=1).items()
         if t is not None}
    t0 = time.perf_counter()
    oracle.gla_forward(f["q"], f["k"], f["v"], f["g"], w.H, w.W, dirs[0], f.get("s0"))
    per_head_call = max(time.perf_counter() - t0, 1e-4)
    total_calls = (args.steps + args.warmup) * len(dirs)
    heads = int(max(1, min(w.heads, 120.0 / (total_calls * per_head_call))))
    spent = 0.0
    for it in range(args.warmup + args.steps):
        for c, d in enumerate(dirs):
            f = {n: t.float().numpy() for n, t in
                 call_inputs(w, d, w.seed(d, 900 + 16 * it + c), heads=heads).items()
                 if t is not None}
            t1 = time.perf_counter()
            oracle.gla_forward(f["q"], f["k"], f["v"], f["g"], w.H, w.W, d, f.get("s0"))
            if it >= args.warmup:
                spent += time.perf_counter() - t1
    frac = heads / w.heads
    tokens = args.steps * len(dirs) * w.B * w.N * frac
    value = tokens / spent
    sample = (f"{heads} of {w.heads} heads of {w.name} per call (tokens scaled by "
              f"{frac:.4f}), {args.steps} timed steps x {len(dirs)} calls, fp64 "
              f"token-by-token oracle, {threads} OpenMP threads")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(spent / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world, "host memory (no GPU L2 involved)",
                                "wall clock of the oracle calls (time.perf_counter)"),
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=400)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=PRIMARY,
                    help="workload timed as the headline (default: the 1.6K-token one)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--sets", type=int, default=None,
                    help="rotating input sets (default: enough to exceed 4x L2); small "
                         "profiler captures use fewer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gate-z", action="store_true",
                    help="time the headline workload through gtr_gla_fwd_z (the gate's "
                         "pre-activation in place of g) instead of gtr_gla_fwd")
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region in this CSV")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
