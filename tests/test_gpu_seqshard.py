"""GPU parity of the sequence-sharded layer's calls (lsa_shard_build_buckets,
lsa_shard_candidates, lsa_shard_merge, lsa_sparse_attn_partial,
lsa_lse_combine) through the C ABI.  The ranks of a job are emulated on one
GPU in one process, one step at a time for every rank (the exchanges are
plain stacks of the ranks' outputs; no kernel waits on another).  Checked:
the union of the ranks' index rows equals lsa_select's rows for the whole
context and the oracle's, segment by segment (bit-exact), and the combined
output is within 2e-2 / 2e-3 of the fp64 oracle (tutorial "隐空间稀疏注意力"
section 二; pages' DCP / CP deployments, news page "开源内容")."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import oracle_cfg, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


def _emulate(lsa, Q, K, V, Wk, Wq, cfg, T, world, chunk):
    from clustered_key_indexing_b200.seqshard import shard_range
    hkv = K.shape[1]
    shards = []
    for r in range(world):
        p0, p1 = shard_range(T, world, r)
        cache = lsa.Cache(hkv, p1 - p0, cfg)
        lsa.shard_build_buckets(K[p0:p1], Wk, cfg, p0, cache)
        shards.append((p0, p1, cache))
    rows, outs = [], []
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        Qc = Q[t0:t0 + n]
        recs = [lsa.shard_candidates(Qc, t0, Wq, c, p0, cfg) for p0, p1, c in shards]
        rec_all = torch.stack([x[0] for x in recs])
        n_all = torch.stack([x[1] for x in recs])
        idxs = [lsa.shard_merge(rec_all, n_all, r, t0, c, p0, cfg) for r, (p0, p1, c) in enumerate(shards)]
        parts = [lsa.sparse_attn_partial(Qc, K[p0:p1], V[p0:p1], idxs[r], p0) for r, (p0, p1, c) in enumerate(shards)]
        outs.append(lsa.lse_combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts])))
        rows.append((t0, [i.cpu().numpy() for i in idxs]))
    torch.cuda.synchronize()
    lsa.check_device_error()
    return torch.cat(outs), rows


def _union_equals(rows, want, S, k):
    for t0, parts in rows:
        for q in range(parts[0].shape[0]):
            for h in range(want.shape[1]):
                w = want[t0 + q, h]
                for lo, hi in ((0, S), (S, S + k), (S + k, w.size)):
                    got = np.concatenate([p[q, h, lo:hi][p[q, h, lo:hi] >= 0] for p in parts])
                    assert np.array_equal(got, w[lo:hi][w[lo:hi] >= 0]), (t0 + q, h, lo)


@pytest.mark.parametrize("name,T,world,agg,chunk", [("prefill-4k", 4096, 2, 0, 1500), ("prefill-4k", 4000, 3, 1, 4000),
                                                     ("decode-small", 4096, 4, 0, 2048)])
def test_sharded_layer_matches_whole_context(lsa, name, T, world, agg, chunk):
    inp = synth.layer_inputs(name, seed=5, T=T)
    c = synth.CONFIGS[name]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=min(c["window"], 300), agg=agg)
    Q, K, V = to_dev_bf16(inp["Q"]), to_dev_bf16(inp["K"]), to_dev_bf16(inp["V"])
    Wk, Wq = to_dev(inp["Wk"]), to_dev(inp["Wq"])
    O, rows = _emulate(lsa, Q, K, V, Wk, Wq, cfg, T, world, chunk)
    # the whole context on one GPU
    cache = lsa.Cache(K.shape[1], T, cfg)
    lsa.build_buckets(K, Wk, cfg, cache)
    idx = lsa.select(Q, 0, Wq, cache, cfg).cpu().numpy()
    _union_equals(rows, idx, cfg.sinks, cfg.k)
    ref = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], oracle_cfg(cfg))
    assert np.array_equal(idx, ref["idx"])
    e = np.abs(O.float().cpu().numpy().astype(np.float64) - ref["O"])
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())


def test_sharded_128k_sampled_rows(lsa):
    """The 128K layer (8 kv-heads, 32 q-heads) over 4 shards: a chunk of
    query positions late in the context, rows against lsa_select's."""
    inp = synth.layer_inputs("prefill-128k", seed=0)
    c = synth.CONFIGS["prefill-128k"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"])
    T = c["T"]
    Q, K, V = to_dev_bf16(inp["Q"]), to_dev_bf16(inp["K"]), to_dev_bf16(inp["V"])
    Wk, Wq = to_dev(inp["Wk"]), to_dev(inp["Wq"])
    from clustered_key_indexing_b200.seqshard import shard_range
    world, t0, n = 4, T - 700, 700
    shards = []
    for r in range(world):
        p0, p1 = shard_range(T, world, r)
        cache = lsa.Cache(8, p1 - p0, cfg)
        lsa.shard_build_buckets(K[p0:p1], Wk, cfg, p0, cache)
        shards.append((p0, p1, cache))
    Qc = Q[t0:t0 + n]
    recs = [lsa.shard_candidates(Qc, t0, Wq, cc, p0, cfg) for p0, p1, cc in shards]
    rec_all, n_all = torch.stack([x[0] for x in recs]), torch.stack([x[1] for x in recs])
    idxs = [lsa.shard_merge(rec_all, n_all, r, t0, cc, p0, cfg).cpu().numpy() for r, (p0, p1, cc) in enumerate(shards)]
    parts = [lsa.sparse_attn_partial(Qc, K[p0:p1], V[p0:p1], to_dev(idxs[r]), p0)
             for r, (p0, p1, cc) in enumerate(shards)]
    O = lsa.lse_combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    cache = lsa.Cache(8, T, cfg)
    lsa.build_buckets(K, Wk, cfg, cache)
    idx = lsa.select(Qc, t0, Wq, cache, cfg)
    O1 = lsa.sparse_attn(Qc, K, V, idx)
    torch.cuda.synchronize()
    lsa.check_device_error()
    full = np.zeros((T, 8, cfg.row), np.int32)
    full[t0:t0 + n] = idx.cpu().numpy()
    _union_equals([(t0, idxs)], full, cfg.sinks, cfg.k)
    e = (O.float() - O1.float()).abs()
    assert e.max().item() <= 2e-2 and e.mean().item() <= 2e-3
