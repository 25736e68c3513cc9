"""The sequence-sharded prefill driver (clustered_key_indexing_b200.seqshard)
on 2 and 3 CPU ranks (gloo, 127.0.0.1): each rank holds a contiguous range
of whole 512-key blocks of the context (the pages' DCP / CP deployments,
news page "开源内容"), the ranks exchange their local fills' records and
their partial attentions with all-gathers, and every rank ends with the
whole layer's output.  The shard steps run as the oracle's fp64 arithmetic
(tests/seqshard_cpu_ops.py); checked against the single-rank oracle: the
union of the ranks' index rows equals the oracle's rows segment by segment
(sinks, long-range keys in order, window), and the outputs agree to 1e-9."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

T = 2600                  # 6 blocks, the last one ragged
CHUNK = 1000


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, agg, out):
    import datetime

    import torch
    import torch.distributed as dist

    import seqshard_cpu_ops
    import synth
    from clustered_key_indexing_b200 import seqshard
    from clustered_key_indexing_b200.api import Config
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        inp = synth.layer_inputs("decode-small", seed=0, T=T)   # 2 kv-heads, 8 query heads
        cfg = Config(k=256, sinks=4, window=300, agg=agg)
        p0, p1 = seqshard.shard_range(T, world, rank)

        def t(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

        ops = seqshard_cpu_ops.OracleOps(inp["Wk"], inp["Wq"], G=4)
        rows = []
        O = seqshard.prefill(t(inp["Q"]), t(inp["K"][p0:p1]), t(inp["V"][p0:p1]), None, None, cfg, T, world, rank,
                             seqshard.torch_all_gather(), ops, chunk=CHUNK, idx_out=rows)
        out[rank] = dict(O=O.numpy(), rows=[(t0, r.numpy()) for t0, r in rows], p=(p0, p1))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,agg", [(2, 0), (3, 1)])
def test_sequence_sharded_prefill_equals_single_rank_oracle(world, agg):
    import oracle
    import synth
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, agg, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    inp = synth.layer_inputs("decode-small", seed=0, T=T)
    ocfg = oracle.Cfg(k=256, sinks=4, window=300, agg=agg)
    ref = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], ocfg)
    S, k = ocfg.sinks, ocfg.k
    assert [res[r]["p"] for r in range(world)][0][0] == 0 and res[world - 1]["p"][1] == T
    for r in range(world):
        assert np.abs(res[r]["O"] - ref["O"]).max() <= 1e-9, r
    for ci, (t0, _) in enumerate(res[0]["rows"]):
        parts = [res[r]["rows"][ci][1] for r in range(world)]
        n = parts[0].shape[0]
        for q in range(n):
            for h in range(ref["idx"].shape[1]):
                want = ref["idx"][t0 + q, h]
                for lo, hi in ((0, S), (S, S + k), (S + k, want.size)):
                    got = np.concatenate([p[q, h, lo:hi][p[q, h, lo:hi] >= 0] for p in parts])
                    w = want[lo:hi][want[lo:hi] >= 0]
                    assert np.array_equal(got, w), (t0 + q, h, lo)
