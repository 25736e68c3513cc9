"""lsa_select_noalloc -- selection for callers that cannot allocate device
memory -- checked through the C ABI against lsa_select (which takes a
caller-allocated workspace), on two calls in a row, in flat and tree mode,
group-mean and native scoring; and its refusals of requests larger than its
built-in scratch.  The file name makes pytest collect it last."""
import ctypes

import pytest
import torch

import synth
from gpu_util import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as lsa
    T = 9000
    inp = synth.layer_inputs("prefill-128k", seed=2, T=T)
    return lsa, T, to_dev_bf16(inp["Q"]), to_dev_bf16(inp["K"]), to_dev(inp["Wk"]), to_dev(inp["Wq"])


def _call(L, Q, t0, n, Wq, cache, tree, cfg, out, stream):
    return L.lsa_select_noalloc(ctypes.c_void_p(Q[t0:t0 + n].data_ptr()), t0, n, 32, ctypes.c_void_p(Wq.data_ptr()),
                                ctypes.byref(cache.c), ctypes.byref(tree.t) if tree is not None else None,
                                ctypes.byref(cfg.c()), ctypes.c_void_p(out.data_ptr()), stream)


@pytest.mark.parametrize("mode,agg", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_noalloc_select_matches_workspace_select_twice(setup, mode, agg):
    from clustered_key_indexing_b200._lib import LSA_OK, lib
    lsa, T, Q, K, Wk, Wq = setup
    L = lib()
    cfg = lsa.Config(k=2048, sinks=4, window=1024, mode=mode, agg=agg)
    cache = lsa.Cache(8, T, cfg)
    lsa.build_buckets(K, Wk, cfg, cache)
    tree = lsa.build_tree(cache, cfg) if mode == 1 else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row over different query ranges: the shared scratch
    # keeps the previous call's contents and must not leak into the next
    for t0, n in ((T - 300, 300), (1500, 257)):
        ref = lsa.select(Q[t0:t0 + n], t0, Wq, cache, cfg, tree=tree)
        out = torch.full_like(ref, -7)
        st = _call(L, Q, t0, n, Wq, cache, tree, cfg, out, stream)
        assert st == LSA_OK, L.lsa_last_error()
        torch.cuda.synchronize()
        lsa.check_device_error()
        assert torch.equal(out, ref), (t0, n)


def test_noalloc_refuses_requests_beyond_its_scratch(setup):
    """A query range whose scratch exceeds the built-in array is refused
    before any work, with the advice to split it; a cache too large for even
    one query's flat search is refused with a message saying so."""
    from clustered_key_indexing_b200._lib import LSA_ENOSPACE, lib
    lsa, T, Q, K, Wk, Wq = setup
    L = lib()
    cfg = lsa.Config(k=2048, sinks=4, window=1024)
    cache = lsa.Cache(8, T, cfg)
    lsa.build_buckets(K, Wk, cfg, cache)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    big = T   # 9000 queries: the candidate lists alone need 9000 x 8 x 8 KB
    assert L.lsa_select_workspace_bytes(ctypes.byref(cfg.c()), big, 32, ctypes.byref(cache.c)) > \
        L.lsa_select_noalloc_scratch_bytes()
    out = torch.empty((big, 8, cfg.row), dtype=torch.int32, device="cuda")
    assert _call(L, Q, 0, big, Wq, cache, None, cfg, out, stream) == LSA_ENOSPACE
    assert b"split the queries" in L.lsa_last_error()
    # a 1M-token cache (8 kv-heads): flat search needs more than the scratch
    # for a single query (the cache is never built: the call refuses first)
    huge = lsa.Cache(8, 1 << 20, cfg)
    huge.c.n_tokens = 1 << 20
    one = torch.empty((1, 8, cfg.row), dtype=torch.int32, device="cuda")
    assert _call(L, Q, 5000, 1, Wq, huge, None, cfg, one, stream) == LSA_ENOSPACE
    assert b"cache is too large" in L.lsa_last_error()
    torch.cuda.synchronize()
