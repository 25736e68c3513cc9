"""GPU parity of batched decode at the benchmark's full size: 32 requests of
2^20 tokens, 8 kv-heads, 32 q-heads, prompts and steps drawn exactly as the
benchmark draws them, steps run in its launch configuration (one
lsa_decode_step per token for the whole batch).

The oracle redoes sampled (request, kv-head) pairs one by one: it clusters
the blocks complete at the decode position (essay "《卡片柜》" ch. 2), selects
for the new query (ch. 3-4) and attends over keys 0..t (tutorial
"隐空间稀疏注意力" section 二).  Checked: index rows bit-exact, outputs
within max |err| 2e-2 / mean |err| 2e-3, at the first step, at the step that
appends the last key of a block (the streaming Ward pass) and after it."""
import numpy as np
import pytest
import torch

import bench
import oracle
import oracle_jobs
import synth
from gpu_util import bits, oracle_cfg

pytestmark = pytest.mark.gpu

WARMUP, STEPS = 3, 5           # the benchmark's warm-up and timed steps of a short decode run
PAIRS = ((0, 0), (31, 7), (17, 3))   # sampled (request, kv-head)


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


def test_decode_32x1m_sampled(lsa):
    from clustered_key_indexing_b200._lib import check, lib
    import ctypes
    c = synth.CONFIGS["decode-32x1m"]
    B, hkv, hq, T = c["batch"], c["hkv"], c["hq"], c["T"]
    G = hq // hkv
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"], mode=c["mode"],
                     agg=c["agg"])
    ocfg = oracle_cfg(cfg)
    # step WARMUP + STEPS // 2 appends key T - 1 (the last key of a block)
    n0, nsteps, cap = bench.decode_plan(T, WARMUP, STEPS)
    assert n0 + WARMUP + STEPS // 2 == T - 1
    dev = torch.device("cuda")
    dec = lsa.Decode(B, hkv, hq, cap, cfg, device=dev)
    Wk_np, Wq_np = synth.projections(0, c["d"], c["dl"])
    Wk, Wq = torch.from_numpy(Wk_np).to(dev), torch.from_numpy(Wq_np).to(dev)
    q, kk, vv = synth.device_decode(c, 0, dev, n0, nsteps, dec.K, dec.V)
    # the oracle's copies of the sampled prompts, taken before any library call
    Kh = {p: bits(dec.K[p[0], :n0, p[1]:p[1] + 1]) for p in PAIRS}
    Vh = {p: bits(dec.V[p[0], :n0, p[1]:p[1] + 1]) for p in PAIRS}
    for r in range(B):
        check(lib().lsa_decode_load(ctypes.byref(dec.d), r, n0, ctypes.c_void_p(Wk.data_ptr()),
                                    ctypes.byref(cfg.c()), ctypes.c_void_p(dec.ws.data_ptr()),
                                    dec.ws.numel(), None), "lsa_decode_load")
    idx = torch.empty((B, hkv, cfg.row), dtype=torch.int32, device=dev)
    o = torch.empty((B, hq, c["d"]), dtype=torch.bfloat16, device=dev)
    qs, ks, vs = bits(q), bits(kk), bits(vv)
    for p in PAIRS:   # append the steps' keys / values to the oracle's copies
        r, h = p
        Kh[p] = np.concatenate([Kh[p], ks[:, r, h:h + 1]])
        Vh[p] = np.concatenate([Vh[p], vs[:, r, h:h + 1]])
    check_at = (0, WARMUP + STEPS // 2, nsteps - 1)
    caches = {}
    for s in range(nsteps):
        dec.step(q[s], kk[s], vv[s], Wk, Wq, o=o, idx_out=idx)
        if s not in check_at:
            continue
        torch.cuda.synchronize()
        lsa.check_device_error()
        t = n0 + s
        g_idx = idx.cpu().numpy()
        g_o = o.float().cpu().numpy().astype(np.float64)
        tb = 512 * ((t + 1) // 512)
        tb_last = 512 * ((n0 + nsteps) // 512)
        for p in PAIRS:
            r, h = p
            if p not in caches:   # every block complete by the last step, clustered once
                U = oracle.key_latent_pool(Kh[p][:tb_last], Wk_np, 4)
                caches[p] = oracle.build_cache(U, tb_last, ocfg)
            oc = oracle_jobs.first_blocks(caches[p], tb)
            Qt = np.ascontiguousarray(qs[s, r:r + 1, G * h:G * (h + 1)])
            Y = oracle.query_latent(Qt, Wq_np, 1, cfg.agg)
            oidx, _, _ = oracle.select(oc, Y, np.array([t]), ocfg, G=G)
            assert np.array_equal(g_idx[r, h], oidx[0, 0]), (s, p, t)
            ref = oracle.attention(Qt, Kh[p][:t + 1], Vh[p][:t + 1], oidx)[0]
            e = np.abs(g_o[r, G * h:G * (h + 1)] - ref)
            assert e.max() <= 2e-2 and e.mean() <= 2e-3, (s, p, e.max(), e.mean())
    assert dec.len == [n0 + nsteps] * B
    del dec
    torch.cuda.empty_cache()


# ------------------------------------------------ 4 x 10M, shared prefix

C5_WARMUP, C5_STEPS = 3, 256       # the benchmark's long-decode run (prompt and prefix lengths follow from it)
C5_PAIRS = ((0, 2), (3, 6))        # sampled (request, kv-head)


def test_decode_4x10m_sampled(lsa, tmp_path):
    """4 requests of 10M tokens sharing one 9,998,848-token prefix (one K/V
    read by every request, each with its own tail), flat search and tree
    search (beam 2), drawn and run as the benchmark's long-decode run draws
    and runs them.  Two (request, kv-head) pairs are redone by the oracle at
    the first step, at the step that appends the last key of a block (the
    streaming Ward pass over a block of the request's own tail) and at the
    step after it: index rows bit-exact, outputs within 2e-2 / 2e-3."""
    import ctypes
    import multiprocessing as mp
    from clustered_key_indexing_b200._lib import check, lib
    c = synth.CONFIGS["decode-4x10m"]
    B, hkv, hq, T = c["batch"], c["hkv"], c["hq"], c["T"]
    G = hq // hkv
    n0, nsteps, cap = bench.decode_plan(T, C5_WARMUP, C5_STEPS)
    sl = 512 * ((n0 - 512) // 512)
    assert sl == 9_998_848
    # steps run: the first, the one appending the last key of a block, the next
    s_blk = next(s for s in range(nsteps) if (n0 + s + 1) % 512 == 0)
    check_at = (0, s_blk, s_blk + 1)
    run_to = s_blk + 2
    dev = torch.device("cuda")
    Wk_np, Wq_np = synth.projections(0, c["d"], c["dl"])
    Wk, Wq = torch.from_numpy(Wk_np).to(dev), torch.from_numpy(Wq_np).to(dev)
    shared = synth.device_shared_prefix(c, 0, dev, sl)

    def fresh(mode):
        cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"], mode=mode,
                         agg=c["agg"])
        dec = lsa.Decode(B, hkv, hq, cap, cfg, device=dev, shared=shared)
        q, kk, vv = synth.device_decode_tails(c, 0, dev, sl, n0, nsteps, dec.K, dec.V)
        return cfg, dec, q, kk, vv

    # the oracle's copies of the sampled contexts (prefix, tail, the steps'
    # keys and values), taken before any library call; one spawned process
    # per pair redoes its context while the library runs
    cfg, dec, q, kk, vv = fresh(0)
    qs, ks, vs = bits(q[:run_to]), bits(kk[:run_to]), bits(vv[:run_to])
    jobs = []
    for p in C5_PAIRS:
        r, h = p
        Kh = np.concatenate([bits(shared[0][:, h:h + 1]), bits(dec.K[r, :n0 - sl, h:h + 1]), ks[:, r, h:h + 1]])
        Vh = np.concatenate([bits(shared[1][:, h:h + 1]), bits(dec.V[r, :n0 - sl, h:h + 1]), vs[:, r, h:h + 1]])
        kp, vp = str(tmp_path / f"K_{r}_{h}.npy"), str(tmp_path / f"V_{r}_{h}.npy")
        np.save(kp, Kh)
        np.save(vp, Vh)
        del Kh, Vh
        jobs.append(dict(K=kp, V=vp, Wk=Wk_np, Wq=Wq_np, G=G, modes=(0, 1),
                         cfg=dict(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"], agg=c["agg"]),
                         queries=[(s, n0 + s, np.ascontiguousarray(qs[s, r:r + 1, G * h:G * (h + 1)]))
                                  for s in check_at]))
    with mp.get_context("spawn").Pool(len(jobs)) as pool:
        pending = pool.map_async(oracle_jobs.decode_context_rows, jobs)
        results = {}
        for mode in (0, 1):
            if mode == 1:
                cfg, dec, q, kk, vv = fresh(1)
            for r in range(B):
                check(lib().lsa_decode_load(ctypes.byref(dec.d), r, n0, ctypes.c_void_p(Wk.data_ptr()),
                                            ctypes.byref(cfg.c()), ctypes.c_void_p(dec.ws.data_ptr()),
                                            dec.ws.numel(), None), "lsa_decode_load")
            idx = torch.empty((B, hkv, cfg.row), dtype=torch.int32, device=dev)
            o = torch.empty((B, hq, c["d"]), dtype=torch.bfloat16, device=dev)
            for s in range(run_to):
                dec.step(q[s], kk[s], vv[s], Wk, Wq, o=o, idx_out=idx)
                if s in check_at:
                    torch.cuda.synchronize()
                    lsa.check_device_error()
                    results[(mode, s)] = (idx.cpu().numpy(), o.float().cpu().numpy().astype(np.float64))
            assert dec.len == [n0 + run_to] * B
            del dec, q, kk, vv, idx, o
            torch.cuda.empty_cache()
        refs = dict(zip(C5_PAIRS, pending.get()))
    del shared
    torch.cuda.empty_cache()
    for (r, h), ref in refs.items():
        for (mode, s), (oidx, oO) in ref.items():
            g_idx, g_o = results[(mode, s)]
            assert np.array_equal(g_idx[r, h], oidx), (mode, s, r, h)
            e = np.abs(g_o[r, G * h:G * (h + 1)] - oO)
            assert e.max() <= 2e-2 and e.mean() <= 2e-3, (mode, s, r, h, e.max(), e.mean())
