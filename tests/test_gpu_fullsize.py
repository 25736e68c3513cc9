"""GPU parity at the benchmark's full sizes, in the benchmark's launch
configuration (same inputs, query chunk, workspaces and call sequence:
lsa_build_buckets, lsa_build_tree, then per query chunk lsa_select followed
by lsa_select_attn).

The oracle cannot redo a whole 1M-token layer in seconds, so it checks
samples it can compute one by one:

* one kv-head's whole bucket cache (and tree), bit-exact: the oracle
  clusters that head's keys alone (Ward per 512-key block, essay "《卡片柜》"
  ch. 2);
* the index rows of that head for 128 sampled query positions in each of
  the first chunk, a middle chunk and the ragged last chunk (first and last
  row of each chunk included), bit-exact (ch. 3-4);
* the attention output of the head's GQA group at those positions, within
  max |err| 2e-2 and mean |err| 2e-3 of the fp64 oracle (tutorial
  "隐空间稀疏注意力" section 二).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bits, oracle_cfg

pytestmark = pytest.mark.gpu

ATOL_MAX, ATOL_MEAN = 2e-2, 2e-3
BENCH_CHUNK = 16384   # the benchmark's requested query chunk
CACHE_KEYS = ("bucket_of_unit", "members", "offsets", "cnt_lr", "minlr", "maxpos")


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


def _cfg(lsa, c):
    return lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"], mode=c["mode"],
                      agg=c["agg"])


class Layer:
    """One workload's device inputs and the oracle's view of kv-heads."""

    def __init__(self, name, device_drawn):
        c = dict(synth.CONFIGS[name])
        self.c = c
        dev = torch.device("cuda")
        if device_drawn:
            self.Q, self.K, self.V = synth.device_layer(c, 0, dev)
            self.Wk_np, self.Wq_np = synth.projections(0, c["d"], c["dl"])
        else:
            inp = synth.layer_inputs(name, seed=0)
            self.Q, self.K, self.V = (torch.from_numpy(inp[x].view(np.int16)).view(torch.bfloat16).to(dev)
                                      for x in "QKV")
            self.Wk_np, self.Wq_np = inp["Wk"], inp["Wq"]
        self.Wk = torch.from_numpy(self.Wk_np).to(dev)
        self.Wq = torch.from_numpy(self.Wq_np).to(dev)
        self._heads = {}

    def head(self, h, ocfg):
        """(K, V, U, oracle cache) of kv-head h, from the input bytes."""
        if h not in self._heads:
            K1 = bits(self.K[:, h:h + 1])
            V1 = bits(self.V[:, h:h + 1])
            U = oracle.key_latent_pool(K1, self.Wk_np, 4)
            oc = oracle.build_cache(U, self.c["T"], ocfg)
            self._heads[h] = (K1, V1, U, oc)
        return self._heads[h]


def _assert_head_cache(cache, h, U, oc):
    """Kv-head h of the library's cache equals the oracle's cache (1 head)."""
    NB = oc["NB"]
    NU = U.shape[1]
    g = dict(
        bucket_of_unit=cache.bucket_of_unit[h, :NU], members=cache.members[h, :NU],
        offsets=cache.offsets[h, :NB + 1], cnt_lr=cache.cnt_lr[h, :NB], minlr=cache.minlr[h, :NB],
        maxpos=cache.maxpos[h, :NB])
    for key in CACHE_KEYS:
        assert np.array_equal(g[key].cpu().numpy(), oc[key][0]), key
    assert np.array_equal(cache.U[h, :NU].cpu().numpy().view(np.uint64), U[0].view(np.uint64))
    assert np.array_equal(cache.sum[h, :NB].cpu().numpy().view(np.uint64), oc["sum"][0].view(np.uint64))
    assert np.array_equal(bits(cache.cent[h, :NB]), oc["cent"][0])
    # packed member words: count in bits 28..30, unit-in-block ids 7 bits each
    pk = cache.units[h, :NB].cpu().numpy().astype(np.int64)
    cnt = (pk >> 28) & 7
    off = oc["offsets"][0]
    assert np.array_equal(cnt, np.diff(off))
    blk = (np.arange(NB) // 64) * 128
    for i in range(4):
        m = cnt > i
        got = blk[m] + ((pk[m] >> (7 * i)) & 127)
        assert np.array_equal(got, oc["members"][0][off[:-1][m] + i]), i


def _run_sampled(lsa, L, cfg, heads, n_per_chunk=128, seed=0):
    """Run the benchmark's launch sequence on three chunks and check sampled
    rows of `heads` against the oracle."""
    c = L.c
    T, hkv, hq = c["T"], c["hkv"], c["hq"]
    G = hq // hkv
    ocfg = oracle_cfg(cfg)
    cache = lsa.Cache(hkv, T, cfg)
    tree = lsa.Tree(cache) if cfg.mode == 1 else None
    lsa.build_buckets(L.K, L.Wk, cfg, cache)
    if tree is not None:
        lsa.build_tree(cache, cfg, tree)
    chunk = lsa.prefill_chunk(cfg, T, hq, hkv, BENCH_CHUNK)
    chunks = [(t0, min(chunk, T - t0)) for t0 in range(0, T, chunk)]
    assert chunks[-1][1] < chunk or T % chunk == 0
    idx = torch.empty((chunk, hkv, cfg.row), dtype=torch.int32, device="cuda")
    O = torch.empty((chunk, hq, 128), dtype=torch.bfloat16, device="cuda")
    sws = torch.empty(lsa.select_workspace_bytes(cfg, chunk, hq, cache) or 1, dtype=torch.uint8, device="cuda")
    aws = torch.empty(lsa.select_attn_workspace_bytes(chunk, hq) or 1, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    lsa.check_device_error()
    for h in heads:
        K1, V1, U, oc = L.head(h, ocfg)
        _assert_head_cache(cache, h, U, oc)
        if tree is not None:
            ot = oracle.build_tree(oc)
            for lvl, (n, off) in enumerate(zip(ot["level_n"], ot["level_off"])):
                goff = tree.level_off[lvl]
                assert np.array_equal(tree.minlr[h, goff:goff + n].cpu().numpy(), ot["minlr"][0, off:off + n])
                assert np.array_equal(bits(tree.cent[h, goff:goff + n]), ot["cent"][0, off:off + n])
    rng = np.random.default_rng(seed)
    for t0, n in (chunks[0], chunks[len(chunks) // 2], chunks[-1]):
        lsa.select(L.Q[t0:t0 + n], t0, L.Wq, cache, cfg, tree=tree, idx=idx[:n], ws=sws)
        lsa.select_attn(L.Q[t0:t0 + n], L.K, L.V, idx[:n], t0, cfg, T, O=O[:n], ws=aws)
        torch.cuda.synchronize()
        lsa.check_device_error()
        rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(n, n_per_chunk), replace=False)]))
        tpos = t0 + rows
        g_idx = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
        g_O = O[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
        Qs = bits(L.Q[torch.from_numpy(tpos).cuda()])
        for h in heads:
            K1, V1, U, oc = L.head(h, ocfg)
            ot = oracle.build_tree(oc) if cfg.mode == 1 else None
            Qh = np.ascontiguousarray(Qs[:, G * h:G * (h + 1)])
            Y = oracle.query_latent(Qh, L.Wq_np, 1, cfg.agg)
            oidx, _, _ = oracle.select(oc, Y, tpos, ocfg, tree=ot, G=G)
            assert np.array_equal(g_idx[:, h], oidx[:, 0]), (t0, h)
            ref = oracle.attention(Qh, K1, V1, oidx)
            e = np.abs(g_O[:, G * h:G * (h + 1)] - ref)
            assert e.max() <= ATOL_MAX and e.mean() <= ATOL_MEAN, (t0, h, e.max(), e.mean())


@pytest.fixture(scope="module")
def layer_1m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = Layer("prefill-1m", device_drawn=True)
    yield L
    del L
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def layer_128k():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = Layer("prefill-128k", device_drawn=False)
    yield L
    del L
    torch.cuda.empty_cache()


@pytest.mark.parametrize("agg", [0, 1])
def test_prefill_128k_sampled(lsa, layer_128k, agg):
    """128K tokens, 8 kv-heads, 32 q-heads: group-mean and native (max over
    the group's heads) scoring, kv-heads 0 and 7."""
    cfg = _cfg(lsa, dict(layer_128k.c, agg=agg))
    _run_sampled(lsa, layer_128k, cfg, heads=(0, 7), seed=agg)


def test_prefill_1m_flat_sampled(lsa, layer_1m):
    """2^20 tokens, flat search (the wave-aligned multi-chunk candidate path),
    kv-heads 1 and 5."""
    cfg = _cfg(lsa, layer_1m.c)
    _run_sampled(lsa, layer_1m, cfg, heads=(1, 5), seed=1)


def test_prefill_1m_tree_sampled(lsa, layer_1m):
    """2^20 tokens, tree search with beam 2, kv-heads 1 and 5."""
    cfg = _cfg(lsa, dict(layer_1m.c, mode=1))
    _run_sampled(lsa, layer_1m, cfg, heads=(1, 5), seed=2)


def test_prefill_128k_exact_fallback(lsa, layer_128k):
    """The exact fallback at full size.  Two kv-heads of the 128K layer are
    replaced: kv-head 3's keys are all zero (every centroid is 0, so every
    eligible bucket ties at score 0 and the candidate list overflows) and
    kv-head 6's keys are 4 x one of three centres, with no noise (few
    distinct scores, so wide bands of exactly tied buckets at the cut).  Rows
    whose ranking the tensor-core scores cannot settle take the exact fp64
    fallback kernel; their index rows must still equal the oracle's bit for
    bit, and the fallback must have run."""
    from clustered_key_indexing_b200._lib import lib
    base = layer_128k
    c = base.c
    L = Layer.__new__(Layer)
    L.c, L.Q, L.V, L.Wk, L.Wq, L.Wk_np, L.Wq_np = base.c, base.Q, base.V, base.Wk, base.Wq, base.Wk_np, base.Wq_np
    L._heads = {}
    K = base.K.clone()
    K[:, 3] = 0
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    mu = torch.from_numpy(synth.centres(0, c["n_centres"], c["d"])[:3]).cuda()
    ci = torch.randint(0, 3, (c["T"],), generator=gen, device="cuda")
    K[:, 6] = (4.0 * mu[ci]).to(torch.bfloat16)
    L.K = K
    cfg = _cfg(lsa, c)
    lib().lsa_fallback_rows()  # reset the counter
    _run_sampled(lsa, L, cfg, heads=(3, 6, 0), n_per_chunk=64, seed=3)
    assert lib().lsa_fallback_rows() > 0
    del L, K
    torch.cuda.empty_cache()
