"""The multi-rank host logic of bench.py and the kv-head split on CPU ranks (gloo, 127.0.0.1).

The LSA layer shards without a data-path collective: each rank takes hkv / N
kv-heads of the layer (decode: a slice of the requests), so the only
cross-rank steps of the benchmark are the timing reduction and the job
throughput.  Checked here: every rank gets the slowest rank's time, the job
rate counts every rank's units at that time, ranks draw distinct inputs, the
reference arm does no work off rank 0, the head and request ranges partition
the layer, and a two-rank kv-head split (the oracle's arithmetic per rank)
reproduces the whole layer's output.
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


def test_head_and_request_ranges_partition():
    from clustered_key_indexing_b200.shard import head_range, request_range
    for world in (1, 2, 4, 8):
        spans = [head_range(8, 32, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == 8 and spans[-1][3] == 32
        for (h0, h1, q0, q1), nxt in zip(spans, spans[1:] + [None]):
            assert q0 == 4 * h0 and q1 == 4 * h1
            if nxt:
                assert h1 == nxt[0] and q1 == nxt[2]
    for world in (1, 3, 5, 32):
        rr = [request_range(32, world, r) for r in range(world)]
        assert rr[0][0] == 0 and rr[-1][1] == 32 and all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
        assert max(b - a for a, b in rr) - min(b - a for a, b in rr) <= 1
    with pytest.raises(ValueError):
        head_range(8, 32, 3, 0)


def _head_rank(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from clustered_key_indexing_b200.shard import head_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T = 1500
        inp = synth.layer_inputs("decode-small", seed=3, T=T)   # 2 kv-heads, 8 query heads
        h0, h1, q0, q1 = head_range(2, 8, world, rank)
        cfg = oracle.Cfg(k=256, sinks=4, window=300)
        res = oracle.layer(inp["Q"][:, q0:q1], inp["K"][:, h0:h1], inp["V"][:, h0:h1], inp["Wk"], inp["Wq"], cfg)
        O = torch.from_numpy(np.ascontiguousarray(res["O"]))
        parts = [torch.empty_like(O) for _ in range(world)]
        dist.all_gather(parts, O)
        out[rank] = torch.cat(parts, dim=1).numpy()
    finally:
        dist.destroy_process_group()


def test_kv_head_split_equals_whole_layer():
    """Two ranks each run the layer for one of the two kv-heads (and its four
    query heads); the outputs, gathered in rank order, are the whole layer's."""
    import oracle
    import synth
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_head_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    inp = synth.layer_inputs("decode-small", seed=3, T=1500)
    ref = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], oracle.Cfg(k=256, sinks=4, window=300))
    for r in range(world):
        assert np.array_equal(res[r], ref["O"])
