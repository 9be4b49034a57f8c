"""Multi-process host logic of the benchmark, on CPU with the gloo backend (world size 2).

Sequences ((batch, head) pairs) are independent, so the data path shards with no
collective: each rank either draws its own batch (the benchmark's weak scaling) or
owns a contiguous slice of one batch.  These tests check the slice bookkeeping,
that the sliced runs reassemble into the full result (checked with the oracle on
the CPU), and the max-over-ranks timing reduction.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        import oracle
        from recurrent_vision_backbone_b200.inputs import make_inputs
        # max-over-ranks timing
        m = bench.max_over_ranks(1.5 * (rank + 1), world, "cpu")
        # one batch split over ranks by sequence (b, h): B=2, heads=3 -> 6 sequences
        B, heads, H, W, dk, dv = 2, 3, 5, 7, 8, 4
        inp = make_inputs(B, heads, H, W, dk, dv, seed=11, init_std=0.2)
        f = {n: t.float().numpy() for n, t in inp.items()}
        seqs = list(bench.shard_sequences(B * heads, world, rank))
        outs = []
        for s in seqs:
            b, h = divmod(s, heads)
            sl = {n: (x[b:b + 1, :, h:h + 1] if n != "s0" else x[b:b + 1, h:h + 1])
                  for n, x in f.items()}
            o, sf = oracle.gla_forward(sl["q"], sl["k"], sl["v"], sl["g"], H, W, 2, sl["s0"])
            outs.append((s, o, sf))
        gathered = [None] * world
        dist.all_gather_object(gathered, outs)
        ok = True
        if rank == 0:
            full_o, full_s = oracle.gla_forward(f["q"], f["k"], f["v"], f["g"], H, W, 2, f["s0"])
            seen = set()
            for part in gathered:
                for s, o, sf in part:
                    b, h = divmod(s, heads)
                    seen.add(s)
                    ok &= np.array_equal(o[0, :, 0], full_o[b, :, h])
                    ok &= np.array_equal(sf[0, 0], full_s[b, h])
            ok &= seen == set(range(B * heads))
        out_q.put((rank, m, ok, seqs, bench.rank_seed(100, rank)))
    finally:
        dist.destroy_process_group()


def test_gloo_world2_sharding_and_timing_reduction():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = {r[0]: r for r in results}
    assert by_rank[0][1] == by_rank[1][1] == 3.0          # max of 1.5 and 3.0
    assert by_rank[0][2] is True                            # sliced runs == full run
    assert by_rank[0][3] + by_rank[1][3] == list(range(6))  # disjoint, complete slices
    assert by_rank[0][4] != by_rank[1][4]                   # independent batches per rank


def test_shard_sequences_cover_every_sequence():
    for n in (1, 5, 16, 128):
        for world in (1, 2, 3, 8):
            got = [s for r in range(world) for s in bench.shard_sequences(n, world, r)]
            assert got == list(range(n))
