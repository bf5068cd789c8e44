"""The N > 1 host logic of bench.py on two gloo ranks (CPU, no GPU).

The forward shards with no data-path collective: each rank draws and runs its own
batch (weak scaling), and the only cross-rank steps are the barrier and the max
of the step time.  This checks those on a real two-process group: the max-over-
ranks reduction, per-rank batches that differ, the whole-job token count, and
that the reference arm works on rank 0 only.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    import datetime

    import numpy as np
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    from hierarchical_fenwick_state_b200 import inputs as I

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = 3.0 + 2.0 * rank                     # rank 1 is the slow one
        worst = bench.max_over_ranks(step_ms, dist, "cpu")
        w = I.shrink(I.WORKLOADS["t2k_d64_bf16"], B=1, H=2, T=64)
        inp = I.make_inputs(w, seed=bench.rank_seed(0, rank))
        digest = float(np.abs(inp.q).sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)

        class Args:
            steps, warmup, seed = 1, 0, 0

        ref_line = bench.run_reference(Args, I.shrink(w, T=32), rank, world)
        # the backward and decoding benches' reference arms follow the same rule
        bwd_line = bench.run_bwd_reference(Args, I.shrink(w, T=32), rank, world)
        dw = I.DecodeWorkload("d", B=2, H=2, L=6, dk=32, dv=32, dtype="f32")
        dec_line = bench.run_decode_reference(Args, dw, rank, world)
        others = [x is None for x in (bwd_line, dec_line)]
        dist.barrier()
        q.put((rank, worst, digests, ref_line is None, ref_line and ref_line["impl"], others))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, worst, digests, ref_none, impl, others = q.get(timeout=120)
        res[rank] = (worst, digests, ref_none, impl, others)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the slowest rank's time is every rank's time
    assert res[0][0] == res[1][0] == 5.0
    # each rank ran a different batch
    assert res[0][1][0] != res[0][1][1]
    # the reference arm prints on rank 0 only; other ranks do no work
    assert res[0][2] is False and res[0][3] == "reference"
    assert res[1][2] is True
    assert res[0][4] == [False, False] and res[1][4] == [True, True]


def test_single_process_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.rank_seed(7, 0) != bench.rank_seed(7, 1)
    assert bench.max_over_ranks(1.25, None, "cpu") == 1.25
