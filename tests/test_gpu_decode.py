"""GPU parity of the batched decode step (lsa_decode_step) against the CPU
oracle: at a decode position t the oracle clusters the blocks complete at t
(streaming, essay "《卡片柜》" ch. 2), selects for query t (ch. 3-4) and
attends over the keys 0..t (tutorial "隐空间稀疏注意力" §二).  Index rows
bit-exact, outputs within max |err| 2e-2 / mean |err| 2e-3."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import oracle_cfg, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

PROMPTS = (1000, 1530, 2047)   # request 2 completes a block on its first step
STEPS = 40


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


@pytest.fixture(scope="module")
def reqs():
    return [synth.layer_inputs("decode-small", seed=r) for r in range(len(PROMPTS))]


def _run_decode(lsa, Kl, Vl, Ql, Wk_np, Wq_np, cfg, shared_len=0, fp8=False):
    """Decode STEPS tokens per request after PROMPTS, checking index rows and
    outputs against the oracle over the logical keys Kl[r] (the shared prefix
    then the request's own tokens).  fp8: the cache keeps FP8 centroids,
    which the flat search scores; the oracle then selects on its own FP8
    centroids (essay ch. 8), and the library's FP8 codes must equal them."""
    c = synth.CONFIGS["decode-small"]
    hkv, hq, cap = c["hkv"], c["hq"], c["T"]
    Wk, Wq = to_dev(Wk_np), to_dev(Wq_np)  # one W_k / W_q per layer
    shared = None
    if shared_len:
        shared = (to_dev_bf16(Kl[0][:shared_len]), to_dev_bf16(Vl[0][:shared_len]))
    dec = lsa.Decode(len(PROMPTS), hkv, hq, cap, cfg, shared=shared, fp8=fp8)
    for r, n in enumerate(PROMPTS):
        dec.load(r, to_dev_bf16(Kl[r][shared_len:n]), to_dev_bf16(Vl[r][shared_len:n]), Wk)
    check_at = {0, 1, 2, 19, STEPS - 1}
    idx = torch.empty((len(PROMPTS), hkv, cfg.row), dtype=torch.int32, device="cuda")
    ocfg = oracle_cfg(cfg)
    caches = {}
    for s in range(STEPS):
        ts = [n + s for n in PROMPTS]
        q = to_dev_bf16(np.stack([Ql[r][t] for r, t in enumerate(ts)]))
        k = to_dev_bf16(np.stack([Kl[r][t] for r, t in enumerate(ts)]))
        v = to_dev_bf16(np.stack([Vl[r][t] for r, t in enumerate(ts)]))
        o = dec.step(q, k, v, Wk, Wq, idx_out=idx)
        completes = any((t + 1) % 512 == 0 or t % 512 == 0 for t in ts)
        if s not in check_at and not completes:
            continue
        torch.cuda.synchronize()
        lsa.check_device_error()
        g_idx = idx.cpu().numpy()
        g_o = o.float().cpu().numpy().astype(np.float64)
        for r, t in enumerate(ts):
            tb = 512 * ((t + 1) // 512)
            key = (r, tb)
            if key not in caches:
                U = oracle.key_latent_pool(Kl[r][:tb], Wk_np, 4)
                oc = oracle.build_cache(U, tb, ocfg)
                caches[key] = (oracle.with_fp8_centroids(oc) if fp8 else oc,
                               oracle.build_tree(oc) if cfg.mode == 1 else None, oc)
            oc, ot, plain = caches[key]
            if fp8:   # the library's FP8 codes of the request's complete blocks
                nb = tb // 512 * 64
                got8 = dec.cache.cent8[r * hkv:(r + 1) * hkv, :nb].cpu().numpy()
                assert np.array_equal(got8, oracle.cent_fp8(plain)), (s, r)
            Qt = Ql[r][t:t + 1]
            Y = oracle.query_latent(Qt, Wq_np, hkv, cfg.agg)
            oidx, _, _ = oracle.select(oc, Y, np.array([t]), ocfg, tree=ot, G=hq // hkv)
            assert np.array_equal(g_idx[r], oidx[0]), (s, r, t)
            ref = oracle.attention(Qt, Kl[r][:t + 1], Vl[r][:t + 1], oidx)[0]
            e = np.abs(g_o[r] - ref)
            assert e.max() <= 2e-2 and e.mean() <= 2e-3, (s, r, e.max(), e.mean())
    assert dec.len == [n + STEPS for n in PROMPTS]


@pytest.mark.parametrize("mode,agg,W", [(0, 0, 600), (0, 1, 600), (1, 0, 600), (1, 1, 600), (0, 0, 128)])
def test_decode_matches_oracle(lsa, reqs, mode, agg, W):
    c = synth.CONFIGS["decode-small"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=W, beam=c["beam"], mode=mode, agg=agg)
    _run_decode(lsa, [x["K"] for x in reqs], [x["V"] for x in reqs], [x["Q"] for x in reqs],
                reqs[0]["Wk"], reqs[0]["Wq"], cfg)


@pytest.mark.parametrize("mode", [0, 1])
def test_decode_shared_prefix_matches_oracle(lsa, reqs, mode):
    """Requests that share their first 512 tokens (read from one shared
    K/V, the pools holding only each request's tail) decode exactly as if
    each held the whole prefix itself."""
    c = synth.CONFIGS["decode-small"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=600, beam=c["beam"], mode=mode, agg=0)
    sl = 512
    Kl = [np.concatenate([reqs[0]["K"][:sl], x["K"][sl:]]) for x in reqs]
    Vl = [np.concatenate([reqs[0]["V"][:sl], x["V"][sl:]]) for x in reqs]
    _run_decode(lsa, Kl, Vl, [x["Q"] for x in reqs], reqs[0]["Wk"], reqs[0]["Wq"], cfg, shared_len=sl)


@pytest.mark.parametrize("agg,shared", [(0, False), (1, False), (0, True)])
def test_decode_fp8_centroids_match_oracle(lsa, reqs, agg, shared):
    """Flat decode over FP8 (e4m3) centroids: the library's codes equal the
    oracle's, and the selection equals the oracle's selection on them, bit
    for bit (products of bf16 and e4m3 values are exact in fp64)."""
    c = synth.CONFIGS["decode-small"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=600, beam=c["beam"], mode=0, agg=agg)
    sl = 512 if shared else 0
    Kl = [np.concatenate([reqs[0]["K"][:sl], x["K"][sl:]]) for x in reqs]
    Vl = [np.concatenate([reqs[0]["V"][:sl], x["V"][sl:]]) for x in reqs]
    _run_decode(lsa, Kl, Vl, [x["Q"] for x in reqs], reqs[0]["Wk"], reqs[0]["Wq"], cfg, shared_len=sl, fp8=True)
