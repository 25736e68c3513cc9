"""lsa_select_noalloc -- selection for callers that cannot allocate device
memory -- checked through the C ABI against lsa_select (which takes a
caller-allocated workspace), on two calls in a row.  The file name makes
pytest collect it last."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from gpu_util import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def test_noalloc_select_matches_workspace_select_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as lsa
    from clustered_key_indexing_b200._lib import LSA_ENOSPACE, LSA_OK, lib

    L = lib()
    T = 9000
    cfg = lsa.Config(k=2048, sinks=4, window=1024)
    inp = synth.layer_inputs("prefill-128k", seed=2, T=T)
    Q, K = to_dev_bf16(inp["Q"]), to_dev_bf16(inp["K"])
    Wk, Wq = to_dev(inp["Wk"]), to_dev(inp["Wq"])
    cache = lsa.Cache(8, T, cfg)
    lsa.build_buckets(K, Wk, cfg, cache)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row over different query ranges: the shared scratch
    # keeps the previous call's contents and must not leak into the next
    for t0, n in ((T - 300, 300), (1500, 257)):
        ref = lsa.select(Q[t0:t0 + n], t0, Wq, cache, cfg)
        out = torch.full_like(ref, -7)
        st = L.lsa_select_noalloc(ctypes.c_void_p(Q[t0:t0 + n].data_ptr()), t0, n, 32,
                                  ctypes.c_void_p(Wq.data_ptr()), ctypes.byref(cache.c), None,
                                  ctypes.byref(cfg.c()), ctypes.c_void_p(out.data_ptr()), stream)
        assert st == LSA_OK, L.lsa_last_error()
        torch.cuda.synchronize()
        lsa.check_device_error()
        assert torch.equal(out, ref), (t0, n)
    # a request larger than the built-in scratch is refused, not run
    big = T
    st = L.lsa_select_noalloc(ctypes.c_void_p(Q.data_ptr()), 0, big, 32, ctypes.c_void_p(Wq.data_ptr()),
                              ctypes.byref(cache.c), None, ctypes.byref(cfg.c()),
                              ctypes.c_void_p(torch.empty((big, 8, cfg.row), dtype=torch.int32,
                                                          device="cuda").data_ptr()), stream)
    need = L.lsa_select_workspace_bytes(ctypes.byref(cfg.c()), big, 32, ctypes.byref(cache.c))
    if need > L.lsa_select_noalloc_scratch_bytes():
        assert st == LSA_ENOSPACE and b"scratch" in L.lsa_last_error()
    else:
        assert st == LSA_OK
