"""Sequence-sharded LSA prefill over the ranks of a job (one process per GPU).

Each rank holds the keys of a contiguous range of whole 512-key cluster
blocks [p0, p1) -- its K/V rows and their bucket cache -- the way the LSA
pages' deployments split the context over GPUs (news page, "开源内容": DCP8
/ CP8 context parallelism).  Every rank sees every query position.  Per
chunk of queries the path takes three local steps and two exchanges:

  candidates   the rank's own flat fill of k keys, as records (global
               bucket id, keys taken, exact score)         [lsa_shard_candidates]
  all-gather   of the records and their counts
  merge        the global fill over all records; the rank's own keys, its
               part of the window, the sinks on the first rank  [lsa_shard_merge]
  partial      exact attention over the rank's own entries -> (O_r, L_r)
                                                            [lsa_sparse_attn_partial]
  all-gather   of the partials, then the log-sum-exp combine [lsa_lse_combine]

Flat search only.  The calls are taken from an `ops` object so that the
same driver runs the library on GPUs (`LibraryOps`, NCCL all-gathers) and,
in the tests, a CPU restatement on gloo ranks.
"""
from __future__ import annotations

import torch

BLOCK = 512


def shard_range(T: int, world: int, rank: int):
    """(p0, p1): the key positions of `rank` -- whole 512-key blocks split as
    evenly as possible in rank order (the last rank's range may end ragged;
    a rank may hold none when there are fewer blocks than ranks)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    nblk = -(-T // BLOCK)
    b0, b1 = rank * nblk // world, (rank + 1) * nblk // world
    return min(T, BLOCK * b0), min(T, BLOCK * b1)


class LibraryOps:
    """The library's calls (CUDA tensors)."""

    def __init__(self, lsa):
        self.lsa = lsa

    def build(self, K_local, W_k, cfg, p0):
        cache = self.lsa.Cache(K_local.shape[1], max(1, K_local.shape[0]), cfg, device=K_local.device)
        if K_local.shape[0] > 0:
            self.lsa.shard_build_buckets(K_local, W_k, cfg, p0, cache)
        return cache

    def cand_cap(self, cfg):
        return self.lsa.shard_cand_cap(cfg)

    def candidates(self, Q, t0, W_q, cache, p0, cfg):
        return self.lsa.shard_candidates(Q, t0, W_q, cache, p0, cfg)

    def merge(self, rec_all, n_all, rank, t0, cache, p0, cfg):
        return self.lsa.shard_merge(rec_all, n_all, rank, t0, cache, p0, cfg)

    def partial(self, Q, K_local, V_local, idx, p0):
        return self.lsa.sparse_attn_partial(Q, K_local, V_local, idx, p0)

    def combine(self, O_all, L_all):
        return self.lsa.lse_combine(O_all, L_all)


def torch_all_gather(group=None):
    """all_gather(x) -> [world, *x.shape] over torch.distributed (NCCL: one
    all_gather_into_tensor; other backends: the list form)."""
    import torch.distributed as dist

    def gather(x):
        world = dist.get_world_size(group)
        x = x.contiguous()
        if dist.get_backend(group) == "nccl":
            out = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
            dist.all_gather_into_tensor(out, x, group=group)
            return out
        parts = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(parts, x, group=group)
        return torch.stack(parts)

    return gather


def prefill(Q, K_local, V_local, W_k, W_q, cfg, T: int, world: int, rank: int, all_gather, ops,
            chunk: int = 4096, idx_out=None):
    """The whole layer over T query positions on one rank of a
    sequence-sharded job: Q [T, hq, 128] (every position), K_local / V_local
    the rank's keys [p1 - p0, hkv, 128].  Returns O [T, hq, 128] (the same on
    every rank).  idx_out: optional list that receives (t0, this rank's index
    rows) per chunk."""
    if cfg.mode != 0:
        raise ValueError("sequence sharding: flat search only")
    p0, p1 = shard_range(T, world, rank)
    if p1 <= p0:
        raise ValueError(f"{T} keys give rank {rank} no 512-key block: use at most {-(-T // BLOCK)} ranks")
    if K_local.shape[0] != p1 - p0:
        raise ValueError(f"rank {rank} holds positions [{p0}, {p1}): K_local must have {p1 - p0} rows")
    cache = ops.build(K_local, W_k, cfg, p0)
    outs = []
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        Qc = Q[t0:t0 + n]
        rec, rec_n = ops.candidates(Qc, t0, W_q, cache, p0, cfg)
        rec_all, n_all = all_gather(rec), all_gather(rec_n)
        idx = ops.merge(rec_all, n_all, rank, t0, cache, p0, cfg)
        if idx_out is not None:
            idx_out.append((t0, idx))
        O_r, L_r = ops.partial(Qc, K_local, V_local, idx, p0)
        outs.append(ops.combine(all_gather(O_r), all_gather(L_r)))
    return torch.cat(outs) if outs else Q.new_empty(Q.shape)
