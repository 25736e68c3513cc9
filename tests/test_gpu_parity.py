"""GPU parity: every stage of the CUDA path (through the C ABI) against the
CPU oracle on the same seeded inputs.

Bar: bucket cache, tree, query latents and index lists bit-exact (the
library takes every quantising or ranking decision on the same fp64 values
as the oracle); attention output within max |err| 2e-2 and mean |err| 2e-3
of the fp64 oracle (bf16 inputs/outputs, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bits, cache_arrays, oracle_cfg, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

CACHE_KEYS = ("bucket_of_unit", "members", "offsets", "cnt_lr", "minlr", "maxpos", "cent")
ATOL_MAX, ATOL_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


def _build_both(lsa, name, T, cfg, seed=0, fp8=False):
    inp = synth.layer_inputs(name, seed=seed, T=T)
    hkv = inp["K"].shape[1]
    K = to_dev_bf16(inp["K"])
    cache = lsa.Cache(hkv, T, cfg, fp8=fp8)
    lsa.build_buckets(K, to_dev(inp["Wk"]), cfg, cache)
    torch.cuda.synchronize()
    lsa.check_device_error()
    U = oracle.key_latent_pool(inp["K"], inp["Wk"], 4)
    oc = oracle.build_cache(U, T, oracle_cfg(cfg))
    return inp, cache, U, oc


def _assert_units_match_members(cache, oc):
    """The packed member-unit words decode to the oracle's CSR members."""
    units = cache.units[:, :oc["NB"]].cpu().numpy()
    for h in range(units.shape[0]):
        for b in range(oc["NB"]):
            pk = int(units[h, b])
            cnt = (pk >> 28) & 7
            got = [(b // 64) * 128 + ((pk >> (7 * i)) & 127) for i in range(cnt)]
            want = oc["members"][h, oc["offsets"][h, b]:oc["offsets"][h, b + 1]].tolist()
            assert got == want, (h, b)


def _assert_cache_equal(cache, U, oc):
    _assert_units_match_members(cache, oc)
    g = cache_arrays(cache, oc["NB"])
    assert np.array_equal(g["U"].view(np.uint64), U.view(np.uint64)), "pooled latents differ"
    assert np.array_equal(g["sum"].view(np.uint64), oc["sum"].view(np.uint64)), "bucket sums differ"
    for key in CACHE_KEYS:
        assert np.array_equal(g[key], oc[key]), key


@pytest.mark.parametrize("T", [4096, 4099, 1000, 513, 512, 7, 4, 1])
def test_build_bit_exact(lsa, T):
    cfg = lsa.Config(k=512, sinks=4, window=256)
    _, cache, U, oc = _build_both(lsa, "prefill-4k", T, cfg)
    _assert_cache_equal(cache, U, oc)


def test_build_bit_exact_8_heads(lsa):
    cfg = lsa.Config(k=2048, sinks=4, window=1024)
    _, cache, U, oc = _build_both(lsa, "prefill-128k", 8192 + 100, cfg)
    _assert_cache_equal(cache, U, oc)


@pytest.mark.parametrize("T", [4096, 1000, 7])
def test_build_fp8_centroids_bit_exact(lsa, T):
    """A cache with FP8 centroids: the e4m3 codes of 2^8 c equal the
    oracle's (essay ch. 8), and the rest of the cache is unchanged."""
    cfg = lsa.Config(k=512, sinks=4, window=256)
    _, cache, U, oc = _build_both(lsa, "prefill-4k", T, cfg, fp8=True)
    _assert_cache_equal(cache, U, oc)
    assert np.array_equal(cache.cent8[:, :oc["NB"]].cpu().numpy(), oracle.cent_fp8(oc))


def test_build_degenerate_keys(lsa):
    """All-zero keys: zero latents, every Delta 0, ties broken by index."""
    cfg = lsa.Config(k=512, sinks=4, window=256)
    T = 1024
    K = np.zeros((T, 1, 128), np.uint16)
    Wk, _ = synth.projections(0)
    cache = lsa.Cache(1, T, cfg)
    lsa.build_buckets(to_dev_bf16(K), to_dev(Wk), cfg, cache)
    torch.cuda.synchronize()
    lsa.check_device_error()
    U = oracle.key_latent_pool(K, Wk, 4)
    oc = oracle.build_cache(U, T, oracle_cfg(cfg))
    _assert_cache_equal(cache, U, oc)


@pytest.mark.parametrize("agg", [0, 1])
def test_query_latent_bit_exact(lsa, agg):
    cfg = lsa.Config(agg=agg)
    inp = synth.layer_inputs("prefill-128k", T=300)
    Y = lsa.query_latent(to_dev_bf16(inp["Q"]), to_dev(inp["Wq"]), 8, cfg)
    torch.cuda.synchronize()
    want = oracle.query_latent(inp["Q"], inp["Wq"], 8, agg)
    assert np.array_equal(bits(Y), want)


def test_tree_bit_exact(lsa):
    cfg = lsa.Config(k=512, sinks=4, window=256, mode=1)
    _, cache, U, oc = _build_both(lsa, "prefill-4k", 4096 + 600, cfg)
    tree = lsa.build_tree(cache, cfg)
    torch.cuda.synchronize()
    ot = oracle.build_tree(oc)
    # the library's tree spans the capacity; it equals the oracle's on every
    # level where the oracle has nodes
    for lvl, (n, off) in enumerate(zip(ot["level_n"], ot["level_off"])):
        goff = tree.level_off[lvl]
        assert np.array_equal(tree.minlr[:, goff:goff + n].cpu().numpy(), ot["minlr"][:, off:off + n])
        assert np.array_equal(bits(tree.cent[:, goff:goff + n]), ot["cent"][:, off:off + n])
        assert np.array_equal(tree.sum[:, goff:goff + n].cpu().numpy().view(np.uint64),
                              ot["sum"][:, off:off + n].view(np.uint64))


def _select_both(lsa, name, T, cfg, tpos=None, seed=0):
    inp, cache, U, oc = _build_both(lsa, name, T, cfg, seed=seed)
    tree = lsa.build_tree(cache, cfg) if cfg.mode == 1 else None
    Q = to_dev_bf16(inp["Q"])
    Wq = to_dev(inp["Wq"])
    idx = lsa.select(Q, 0, Wq, cache, cfg, tree=tree)
    torch.cuda.synchronize()
    lsa.check_device_error()
    hkv, hq = inp["K"].shape[1], inp["Q"].shape[1]
    if tpos is None:
        tpos = np.arange(T)
    Y = oracle.query_latent(inp["Q"][tpos], inp["Wq"], hkv, cfg.agg)
    oidx, mg, nc = oracle.select(oc, Y, tpos, oracle_cfg(cfg), G=hq // hkv)
    return inp, idx.cpu().numpy()[tpos], oidx, mg


@pytest.mark.parametrize("beam,k,agg", [(1, 512, 0), (3, 300, 1), (8, 512, 0)])
def test_tree_beams_bit_exact(lsa, beam, k, agg):
    """Tree search with beam 1 (greedy), 3 (native scores) and 8 (16 children
    scored per level) against the oracle."""
    cfg = lsa.Config(k=k, sinks=4, window=256, mode=1, beam=beam, agg=agg)
    _, g, o, _ = _select_both(lsa, "prefill-4k", 4096, cfg)
    bad = np.where((g != o).any(axis=(1, 2)))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first t={bad[:5]}"


@pytest.mark.parametrize("mode,agg", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_select_bit_exact_4k(lsa, mode, agg):
    cfg = lsa.Config(k=512, sinks=4, window=256, mode=mode, agg=agg)
    _, g, o, _ = _select_both(lsa, "prefill-4k", 4096, cfg)
    bad = np.where((g != o).any(axis=(1, 2)))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first t={bad[:5]}"


@pytest.mark.parametrize("T,k,W", [(1000, 64, 8), (777, 4096, 16), (130, 512, 1), (5, 16, 2)])
def test_select_edge_cases(lsa, T, k, W):
    """Ragged lengths, k above every eligible key (take-all), window 1,
    prompts shorter than the sinks + window."""
    for mode in (0, 1):
        cfg = lsa.Config(k=k, sinks=4, window=W, mode=mode, beam=2)
        _, g, o, _ = _select_both(lsa, "prefill-4k", T, cfg)
        assert np.array_equal(g, o), (mode, np.where((g != o).any(axis=(1, 2)))[0][:5])


def test_select_degenerate_ties(lsa):
    """All-zero keys give all-zero centroids: every score ties and the fill
    takes buckets in ascending id (the band overflow path included)."""
    cfg = lsa.Config(k=64, sinks=4, window=16)
    T = 4096
    K = np.zeros((T, 1, 128), np.uint16)
    inp = synth.layer_inputs("prefill-4k", T=T)
    cache = lsa.Cache(1, T, cfg)
    lsa.build_buckets(to_dev_bf16(K), to_dev(inp["Wk"]), cfg, cache)
    idx = lsa.select(to_dev_bf16(inp["Q"]), 0, to_dev(inp["Wq"]), cache, cfg).cpu().numpy()
    torch.cuda.synchronize()
    lsa.check_device_error()
    oc = oracle.build_cache(oracle.key_latent_pool(K, inp["Wk"], 4), T, oracle_cfg(cfg))
    Y = oracle.query_latent(inp["Q"], inp["Wq"], 1, 0)
    oidx, _, _ = oracle.select(oc, Y, np.arange(T), oracle_cfg(cfg), G=4)
    assert np.array_equal(idx, oidx)


def _attn_err(O_dev, O_ref):
    g = O_dev.float().cpu().numpy().astype(np.float64)
    e = np.abs(g - O_ref)
    return e.max(), e.mean()


def test_sparse_attn_matches_oracle(lsa):
    inp = synth.layer_inputs("prefill-128k", T=3000)
    rng = np.random.default_rng(5)
    nq, n = 96, 700
    idx = rng.integers(0, 3000, size=(nq, 8, n)).astype(np.int32)
    idx[rng.random(idx.shape) < 0.2] = -1
    idx[3, 2, :] = -1                  # an empty list -> zeros
    idx[4, 1, :] = -1
    idx[4, 1, 17] = 123                # a single key -> its value row
    Q = inp["Q"][:nq]
    O = lsa.sparse_attn(to_dev_bf16(Q), to_dev_bf16(inp["K"]), to_dev_bf16(inp["V"]), to_dev(idx))
    torch.cuda.synchronize()
    lsa.check_device_error()
    ref = oracle.attention(Q, inp["K"], inp["V"], idx)
    mx, mean = _attn_err(O, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
    assert np.all(O[3, 8:12].float().cpu().numpy() == 0)


@pytest.mark.parametrize("G,t0,nq,W", [(1, 1500, 700, 300), (2, 0, 333, 300), (4, 900, 515, 1),
                                        (8, 0, 300, 5000)])
def test_select_attn_matches_gather_and_oracle(lsa, G, t0, nq, W):
    """lsa_select_attn (window as a band + gathered sinks / long-range
    entries, merged) against lsa_sparse_attn over the same index rows and
    against the oracle attention: every GQA group size, ragged query ranges,
    windows of 1 and longer than the prompt, queries from position 0."""
    T, hkv = 3000, 2
    inp = synth.layer_inputs("prefill-128k", T=T)
    Q = np.ascontiguousarray(inp["Q"][:, :hkv * G])
    K = np.ascontiguousarray(inp["K"][:, :hkv])
    V = np.ascontiguousarray(inp["V"][:, :hkv])
    cfg = lsa.Config(k=256, sinks=4, window=W)
    dK, dV = to_dev_bf16(K), to_dev_bf16(V)
    cache = lsa.Cache(hkv, T, cfg)
    lsa.build_buckets(dK, to_dev(inp["Wk"]), cfg, cache)
    dQ = to_dev_bf16(Q[t0:t0 + nq])
    idx = lsa.select(dQ, t0, to_dev(inp["Wq"]), cache, cfg)
    O = lsa.select_attn(dQ, dK, dV, idx, t0, cfg, T)
    Og = lsa.sparse_attn(dQ, dK, dV, idx, T)
    torch.cuda.synchronize()
    lsa.check_device_error()
    d = (O.float() - Og.float()).abs()
    assert d.max().item() <= ATOL_MAX and d.mean().item() <= ATOL_MEAN, (d.max().item(), d.mean().item())
    ref = oracle.attention(Q[t0:t0 + nq], K, V, idx.cpu().numpy())
    mx, mean = _attn_err(O, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)


def test_prefill_end_to_end_4k(lsa):
    """The whole layer (lsa_prefill) against the oracle layer."""
    cfg = lsa.Config(k=512, sinks=4, window=256)
    inp = synth.layer_inputs("prefill-4k")
    O = lsa.prefill(to_dev_bf16(inp["Q"]), to_dev_bf16(inp["K"]), to_dev_bf16(inp["V"]),
                    to_dev(inp["Wk"]), to_dev(inp["Wq"]), cfg, chunk=1000)
    torch.cuda.synchronize()
    lsa.check_device_error()
    ref = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], oracle_cfg(cfg))["O"]
    mx, mean = _attn_err(O, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)


def test_prefill_all_keys_is_full_causal_attention(lsa):
    """k >= T: LSA reduces to exact causal attention (torch SDPA in fp32)."""
    T = 2000
    cfg = lsa.Config(k=4096, sinks=4, window=64)
    inp = synth.layer_inputs("prefill-4k", T=T)
    Q, K, V = (to_dev_bf16(inp[x]) for x in "QKV")
    O = lsa.prefill(Q, K, V, to_dev(inp["Wk"]), to_dev(inp["Wq"]), cfg)
    torch.cuda.synchronize()
    q = Q.float().permute(1, 0, 2)
    k = K.float().permute(1, 0, 2).expand(4, T, 128)
    v = V.float().permute(1, 0, 2).expand(4, T, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).permute(1, 0, 2)
    e = (O.float() - ref).abs()
    assert e.max().item() <= ATOL_MAX and e.mean().item() <= ATOL_MEAN


def test_bad_arguments_return_status(lsa):
    from clustered_key_indexing_b200._lib import LSAError, LSA_EINVAL, LSA_EUNSUPPORTED, LSA_ENOSPACE
    cfg = lsa.Config(k=512, sinks=4, window=256)
    inp = synth.layer_inputs("prefill-4k", T=64)
    K = to_dev_bf16(inp["K"])
    small = lsa.Cache(1, 16, cfg)
    with pytest.raises(LSAError) as e:
        lsa.build_buckets(K, to_dev(inp["Wk"]), cfg, small)
    assert e.value.status == LSA_ENOSPACE
    with pytest.raises(LSAError) as e:
        lsa.build_buckets(K, to_dev(inp["Wk"]), lsa.Config(d_latent=32), lsa.Cache(1, 64, cfg))
    assert e.value.status == LSA_EUNSUPPORTED
    with pytest.raises(LSAError) as e:
        lsa.build_buckets(K, to_dev(inp["Wk"]), lsa.Config(window=0), lsa.Cache(1, 64, cfg))
    assert e.value.status == LSA_EINVAL


@pytest.mark.parametrize("mode", [0, 1])
def test_prefill_host_equals_prefill(lsa, mode):
    """lsa_prefill_host (pinned host buffers, overlapped copies on two extra
    streams) gives the bits of lsa_prefill on the same inputs."""
    T = 3000
    cfg = lsa.Config(k=256, sinks=4, window=300, mode=mode)
    inp = synth.layer_inputs("prefill-128k", T=T)
    Qh, Kh, Vh = (np.ascontiguousarray(inp[x][:, :n]) for x, n in (("Q", 8), ("K", 2), ("V", 2)))
    Wk, Wq = to_dev(inp["Wk"]), to_dev(inp["Wq"])
    O_dev = lsa.prefill(to_dev_bf16(Qh), to_dev_bf16(Kh), to_dev_bf16(Vh), Wk, Wq, cfg, chunk=700)
    pin = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (Qh, Kh, Vh)]
    hO = lsa.prefill_host(*pin, Wk, Wq, cfg, chunk=700)
    torch.cuda.synchronize()
    lsa.check_device_error()
    assert torch.equal(hO.view(torch.int16), O_dev.cpu().view(torch.int16))


@pytest.mark.parametrize("scale_q,scale_k", [(2.0 ** -40, 1.0), (1.0, 2.0 ** -40), (2.0 ** -20, 2.0 ** -20)])
def test_tree_exponent_spread_fallback(lsa, scale_q, scale_k):
    """Latents with a component ~2^-40 of the others (one column of W_q or W_k
    scaled) fail the exponent-spread test of the parallel tree descent, so the
    children are scored sequentially; selections stay bit-exact."""
    T = 4096
    cfg = lsa.Config(k=512, sinks=4, window=256, mode=1)
    inp = synth.layer_inputs("prefill-4k", T=T)
    Wk, Wq = inp["Wk"].copy(), inp["Wq"].copy()
    Wk[:, 5] *= np.float32(scale_k)
    Wq[:, 5] *= np.float32(scale_q)
    K, Q = to_dev_bf16(inp["K"]), to_dev_bf16(inp["Q"])
    cache = lsa.Cache(1, T, cfg)
    lsa.build_buckets(K, to_dev(Wk), cfg, cache)
    tree = lsa.build_tree(cache, cfg)
    idx = lsa.select(Q, 0, to_dev(Wq), cache, cfg, tree=tree)
    torch.cuda.synchronize()
    lsa.check_device_error()
    ocfg = oracle_cfg(cfg)
    U = oracle.key_latent_pool(inp["K"], Wk, 4)
    oc = oracle.build_cache(U, T, ocfg)
    tpos = np.arange(0, T, 7)
    Y = oracle.query_latent(inp["Q"][tpos], Wq, 1, 0)
    oidx, _, _ = oracle.select(oc, Y, tpos, ocfg, tree=oracle.build_tree(oc), G=4)
    assert np.array_equal(idx.cpu().numpy()[tpos], oidx)


def test_select_attn_band_with_growing_scores(lsa):
    """Scores that grow along the window by far more than 2^8 per 64-key tile
    move the band kernel's running max on every tile (its rescaling path);
    the output still matches the oracle attention over the same index rows."""
    T, hkv, G, t0, nq = 2100, 1, 4, 1500, 300
    rng = np.random.default_rng(11)
    u = rng.standard_normal(128)
    u /= np.linalg.norm(u)
    pos = np.arange(T, dtype=np.float64)
    K = synth.f32_to_bf16_bits(
        (0.5 * pos)[:, None, None] * u[None, None, :] + 0.05 * rng.standard_normal((T, hkv, 128)))
    V = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 128)))
    Q = synth.f32_to_bf16_bits(4.0 * u[None, None, :] + 0.05 * rng.standard_normal((nq, hkv * G, 128)))
    inp = synth.layer_inputs("prefill-4k", T=T)
    cfg = lsa.Config(k=64, sinks=4, window=1024)
    dK, dV = to_dev_bf16(K), to_dev_bf16(V)
    cache = lsa.Cache(hkv, T, cfg)
    lsa.build_buckets(dK, to_dev(inp["Wk"]), cfg, cache)
    dQ = to_dev_bf16(Q)
    idx = lsa.select(dQ, t0, to_dev(inp["Wq"]), cache, cfg)
    O = lsa.select_attn(dQ, dK, dV, idx, t0, cfg, T)
    torch.cuda.synchronize()
    lsa.check_device_error()
    ref = oracle.attention(Q, K, V, idx.cpu().numpy())
    mx, mean = _attn_err(O, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
