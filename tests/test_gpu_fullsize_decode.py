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

import oracle
import synth
from gpu_util import bits, oracle_cfg

pytestmark = pytest.mark.gpu

WARMUP, STEPS = 3, 5           # the benchmark's default warm-up and timed steps
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
    nsteps = WARMUP + STEPS
    n0 = T - 1 - WARMUP - STEPS // 2       # step WARMUP + STEPS // 2 appends key T - 1
    cap = -(-(n0 + nsteps) // 512) * 512
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
    caches, units = {}, {}
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
        for p in PAIRS:
            r, h = p
            if (p, tb) not in caches:
                if p not in units:   # pooled latents of every whole 4-key unit
                    units[p] = oracle.key_latent_pool(Kh[p][:(len(Kh[p]) // 4) * 4], Wk_np, 4)
                U = np.ascontiguousarray(units[p][:, :tb // 4])
                caches[(p, tb)] = oracle.build_cache(U, tb, ocfg)
            oc = caches[(p, tb)]
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
