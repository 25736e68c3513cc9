"""The multi-rank host logic of bench.py on two CPU ranks (gloo, 127.0.0.1).

The LSA layer shards without a data-path collective (each rank runs its own
layer or decode batch: weak scaling), so the only cross-rank steps are the
timing reduction and the job throughput.  Checked here: every rank gets the
slowest rank's time, the job rate counts every rank's units at that time,
ranks draw distinct inputs, and the reference arm does no work off rank 0.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        rate = bench.job_rate(world, 4096, ms / 2)
        k = synth.layer_inputs("prefill-4k", seed=rank, T=64, parts=("K",))["K"]
        ks = [None] * world
        dist.all_gather_object(ks, k)
        # the reference arm returns at once on every rank but 0
        ref_ran = None
        if rank != 0:
            class A:
                workload = "prefill-4k"
            bench.run_reference(A())
            ref_ran = False
        out[rank] = dict(ms=ms, rate=rate, distinct=not np.array_equal(ks[0], ks[1]), ref_ran=ref_ran)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0]["ms"] == res[1]["ms"] == pytest.approx(15.0)
    assert res[0]["rate"] == pytest.approx(2 * 4096 / (7.5e-3))
    assert res[0]["distinct"] and res[1]["distinct"]
    assert res[1]["ref_ran"] is False
