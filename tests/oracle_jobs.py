"""Oracle work of the GPU tests that runs in spawned worker processes
(numpy and the oracle only; no torch, no CUDA), so that a long oracle build
proceeds while the library runs."""
import numpy as np

import oracle


def first_blocks(oc: dict, tb: int) -> dict:
    """The oracle cache restricted to its first tb keys (tb a multiple of
    512).  Cluster blocks are clustered independently, so this equals the
    cache the oracle builds from those keys alone."""
    nblk = tb // 512
    NU, NB = tb // 4, nblk * 64
    out = dict(oc, T=tb, NU=NU, NB=NB, nblk=nblk)
    for key in ("bucket_of_unit", "members"):
        out[key] = np.ascontiguousarray(oc[key][:, :NU])
    out["offsets"] = np.ascontiguousarray(oc["offsets"][:, :NB + 1])
    for key in ("cnt_lr", "minlr", "maxpos", "sum", "cent"):
        out[key] = np.ascontiguousarray(oc[key][:, :NB])
    out["ward_margin"] = np.ascontiguousarray(oc["ward_margin"][:, :nblk])
    return out


def decode_context_rows(job: dict) -> dict:
    """One (request, kv-head) decode context redone by the oracle: the keys'
    pooled latents, the cache of every block complete at each checked step
    (blocks complete when their last key is appended), the tree where asked,
    the selection for that step's query and the attention over keys 0..t.

    job: K, V (paths of .npy bf16 bits [n, 1, 128]), Wk, Wq, cfg (oracle.Cfg
    fields without mode), modes, G, queries [(step, t, Q rows [1, G, 128])].
    Returns {(mode, step): (index row [S + k + W], O [G, 128] fp64)}."""
    K = np.load(job["K"], mmap_mode="r")
    V = np.load(job["V"], mmap_mode="r")
    tbs = sorted({512 * ((t + 1) // 512) for _, t, _ in job["queries"]})
    U = oracle.key_latent_pool(np.ascontiguousarray(K[:tbs[-1]]), job["Wk"], 4)
    base = oracle.Cfg(**job["cfg"])
    full = oracle.build_cache(U, tbs[-1], base)
    del U
    caches, trees, out = {}, {}, {}
    for s, t, Qt in job["queries"]:
        tb = 512 * ((t + 1) // 512)
        if tb not in caches:
            caches[tb] = first_blocks(full, tb)
        oc = caches[tb]
        Y = oracle.query_latent(Qt, job["Wq"], 1, base.agg)
        for mode in job["modes"]:
            cfg = oracle.Cfg(**dict(job["cfg"], mode=mode))
            ot = None
            if mode == 1:
                if tb not in trees:
                    trees[tb] = oracle.build_tree(oc)
                ot = trees[tb]
            oidx, _, _ = oracle.select(oc, Y, np.array([t]), cfg, tree=ot, G=job["G"])
            ref = oracle.attention(Qt, K[:t + 1], V[:t + 1], oidx)[0]
            out[(mode, s)] = (oidx[0, 0].copy(), ref)
    return out
