"""C ABI checks that need no GPU: liblsa.so loads, exports every function
include/lsa.h declares, and its host-only calls and argument validation
behave as documented (no compute call is made here)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from clustered_key_indexing_b200 import _lib
from clustered_key_indexing_b200._lib import (LSA_EINVAL, LSA_ENOSPACE, LSA_EUNSUPPORTED, LSA_OK,
                                              lsa_cache, lsa_cfg, lsa_decode, lsa_tree)


@pytest.fixture(scope="module")
def L():
    from clustered_key_indexing_b200.build import build
    build()
    return _lib.lib()


def test_every_declared_symbol_is_exported(L):
    names = _lib.exported_names()
    assert len(names) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.SO], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)


def test_defaults_and_checks(L):
    c = lsa_cfg()
    assert L.lsa_cfg_default(ctypes.byref(c)) == LSA_OK
    assert (c.d_head, c.d_latent, c.pool, c.block, c.bucket_mean, c.bucket_max) == (128, 64, 4, 512, 8, 16)
    assert (c.k, c.sinks, c.window, c.beam, c.mode, c.agg) == (2048, 4, 1024, 2, 0, 0)
    assert L.lsa_cfg_check(ctypes.byref(c)) == LSA_OK
    bad = lsa_cfg.from_buffer_copy(c)
    bad.d_latent = 32
    assert L.lsa_cfg_check(ctypes.byref(bad)) == LSA_EUNSUPPORTED
    assert b"d_latent" in L.lsa_last_error()
    bad = lsa_cfg.from_buffer_copy(c)
    bad.window = 0
    assert L.lsa_cfg_check(ctypes.byref(bad)) == LSA_EINVAL
    bad = lsa_cfg.from_buffer_copy(c)
    bad.mode = 3
    assert L.lsa_cfg_check(ctypes.byref(bad)) == LSA_EINVAL
    assert L.lsa_cfg_check(None) == LSA_EINVAL


def test_sizes_and_tree_layout(L):
    c = lsa_cfg()
    L.lsa_cfg_default(ctypes.byref(c))
    assert L.lsa_cache_units(ctypes.byref(c), 4097) == 1025
    assert L.lsa_cache_buckets(ctypes.byref(c), 4096) == 512
    assert L.lsa_cache_buckets(ctypes.byref(c), 4097) == 576
    assert L.lsa_cache_buckets(ctypes.byref(c), 1 << 20) == 131072
    t = lsa_tree()
    assert L.lsa_tree_layout(131072, ctypes.byref(t)) == LSA_OK
    assert t.levels == 18 and t.level_n[17] == 1 and t.n_nodes == 2 * 131072 - 1
    assert L.lsa_tree_layout(5, ctypes.byref(t)) == LSA_OK
    assert [t.level_n[i] for i in range(t.levels)] == [5, 3, 2, 1]
    assert [t.level_off[i] for i in range(t.levels)] == [0, 5, 8, 10]
    assert L.lsa_tree_layout(0, ctypes.byref(t)) == LSA_EINVAL
    cache = lsa_cache(8, 131072, 32768, 16384, *([16] * 10))
    assert L.lsa_select_workspace_bytes(ctypes.byref(c), 131072, 32, ctypes.byref(cache)) > 0
    assert L.lsa_prefill_workspace_bytes(ctypes.byref(c), 131072, 32, 8, 16384) > 0


def test_compute_calls_reject_bad_arguments_before_any_launch(L):
    c = lsa_cfg()
    L.lsa_cfg_default(ctypes.byref(c))
    # NULL cache / NULL tensors / bad head ratio: refused on the host
    assert L.lsa_build_buckets(None, 16, 1, None, ctypes.byref(c), None, None) == LSA_EINVAL
    cache = lsa_cache(1, 0, 4, 64, *([0] * 10))
    assert L.lsa_build_buckets(None, 16, 1, None, ctypes.byref(c), ctypes.byref(cache), None) == LSA_EINVAL
    assert L.lsa_sparse_attn(None, None, None, None, 1, 3, 2, 8, 16, None, None) == LSA_EINVAL
    assert L.lsa_sparse_attn(None, None, None, None, 1, 48, 4, 8, 16, None, None) == LSA_EUNSUPPORTED
    assert L.lsa_query_latent(None, 1, 4, 1, None, ctypes.byref(c), None, None) == LSA_EINVAL
    assert L.lsa_select(None, 0, 1, 4, None, None, None, ctypes.byref(c), None, None, None, 0, None) == LSA_EINVAL
    assert L.lsa_prefill(None, None, None, 16, 4, 1, None, None, ctypes.byref(c), None, None, None, 0,
                         None, 0, None) == LSA_EINVAL


def _fake(addr=0x10000):
    """A non-NULL, 16-byte aligned device address that no call below reaches
    (each is refused on the host before any CUDA call)."""
    return ctypes.c_void_p(addr)


def _decode_state(batch=2, hkv=2, hq=8, cap=1024, shared_len=0):
    d = lsa_decode()
    d.batch, d.hkv, d.hq, d.cap, d.shared_len = batch, hkv, hq, cap, shared_len
    d.K = d.V = d.U_blk = _fake().value
    d.K_shared = d.V_shared = _fake().value if shared_len else None
    c = d.cache
    c.hkv, c.cap_units, c.cap_buckets = batch * hkv, cap // 4, cap // 512 * 64
    for f in ("bucket_of_unit", "members", "offsets", "cnt_lr", "minlr", "maxpos", "sum", "cent", "units"):
        setattr(c, f, _fake().value)
    return d


def _no_gpu():
    import torch
    return not torch.cuda.is_available()


@pytest.mark.skipif(not _no_gpu(), reason="passes fake device addresses: runs only where no GPU is present")
def test_host_buffer_pca_and_decode_calls_reject_bad_arguments(L):
    c = lsa_cfg()
    L.lsa_cfg_default(ctypes.byref(c))
    f = _fake()
    # training-free projection: NULLs, sizes, d_latent range, K alignment, workspace
    assert L.lsa_fit_pca(None, 16, 1, 64, f, None, f, 1 << 30, None) == LSA_EINVAL
    assert L.lsa_fit_pca(f, 0, 1, 64, f, None, f, 1 << 30, None) == LSA_EINVAL
    assert L.lsa_fit_pca(f, 16, 1, 0, f, None, f, 1 << 30, None) == LSA_EINVAL
    assert L.lsa_fit_pca(f, 16, 1, 129, f, None, f, 1 << 30, None) == LSA_EINVAL
    assert L.lsa_fit_pca(_fake(0x10008), 16, 1, 64, f, None, f, 1 << 30, None) == LSA_EINVAL
    assert L.lsa_fit_pca(f, 16, 1, 64, f, None, f, 0, None) == LSA_ENOSPACE
    assert L.lsa_fit_pca_workspace_bytes(16, 1) > 0 and L.lsa_fit_pca_workspace_bytes(0, 1) == 0
    # prefill from host buffers: NULL host / device pointers, T, workspace
    args = [f] * 8
    assert L.lsa_prefill_host(None, f, f, f, *args[4:], 4096, 4, 1, f, f, ctypes.byref(c), None, None,
                              0, f, 1 << 40, None, None, None) == LSA_EINVAL
    assert L.lsa_prefill_host(*args, 4096, 4, 1, None, f, ctypes.byref(c), None, None,
                              0, f, 1 << 40, None, None, None) == LSA_EINVAL
    assert L.lsa_prefill_host(*args, 0, 4, 1, f, f, ctypes.byref(c), None, None,
                              0, f, 1 << 40, None, None, None) == LSA_EINVAL
    assert L.lsa_prefill_host(*args, 4096, 4, 1, f, f, ctypes.byref(c), None, None,
                              0, f, 0, None, None, None) == LSA_ENOSPACE
    # decode: the state's shape, then the call's own arguments
    assert L.lsa_decode_step(None, f, f, f, f, f, ctypes.byref(c), f, None, f, 1 << 40, None) == LSA_EINVAL
    for kw, want in ((dict(batch=0), LSA_EUNSUPPORTED), (dict(hq=6, hkv=4), LSA_EINVAL),
                     (dict(hq=6, hkv=2), LSA_EUNSUPPORTED), (dict(cap=1000), LSA_EINVAL),
                     (dict(shared_len=256), LSA_EINVAL)):
        d = _decode_state(**kw)
        if "cap" in kw:
            d.cache.cap_units, d.cache.cap_buckets = 250, 64
        assert L.lsa_decode_step(ctypes.byref(d), f, f, f, f, f, ctypes.byref(c), f, None, f,
                                 1 << 40, None) == want, kw
    d = _decode_state(shared_len=512)
    d.K_shared = None
    assert L.lsa_decode_load(ctypes.byref(d), 0, 600, f, ctypes.byref(c), f, 1 << 40, None) == LSA_EINVAL
    d = _decode_state()
    d.cache.cent = None
    assert L.lsa_decode_load(ctypes.byref(d), 0, 600, f, ctypes.byref(c), f, 1 << 40, None) == LSA_EINVAL
    d = _decode_state(shared_len=512)
    assert L.lsa_decode_load(ctypes.byref(d), 2, 600, f, ctypes.byref(c), f, 1 << 40, None) == LSA_EINVAL
    assert L.lsa_decode_load(ctypes.byref(d), 0, 1024, f, ctypes.byref(c), f, 1 << 40, None) == LSA_ENOSPACE
    assert L.lsa_decode_load(ctypes.byref(d), 0, 300, f, ctypes.byref(c), f, 1 << 40, None) == LSA_EINVAL
    assert L.lsa_decode_load(ctypes.byref(d), 0, 600, f, ctypes.byref(c), f, 0, None) == LSA_ENOSPACE
    assert L.lsa_decode_workspace_bytes(ctypes.byref(c), ctypes.byref(d)) > 0
    d.len[1] = 1024
    assert L.lsa_decode_step(ctypes.byref(d), f, f, f, f, f, ctypes.byref(c), f, None, f,
                             1 << 40, None) == LSA_ENOSPACE


def test_prefill_chunk_is_whole_waves_of_the_candidate_kernel(L):
    """Host logic: in flat mode the query chunk is a whole number of waves of
    the candidate kernel (512 / G latent rows per CTA, CTAs a multiple of the
    148 SMs), the nearest to the request; tree mode keeps the request."""
    import clustered_key_indexing_b200 as lsa
    for agg, G in ((0, 1), (1, 4)):
        cfg = lsa.Config(k=2048, sinks=4, window=1024, agg=agg)
        for T, hkv, hq in ((131072, 8, 32), (1 << 20, 8, 32), (50000, 2, 8)):
            ch = lsa.prefill_chunk(cfg, T, hq, hkv, 16384)
            if ch == T:
                continue
            rows_per_cta = 512 // (hq // hkv if agg else 1)
            assert ch % rows_per_cta == 0
            assert (ch // rows_per_cta * hkv) % 148 == 0, (agg, T, ch)
            wave = rows_per_cta * 148 // np.gcd(148, hkv)
            assert abs(ch - 16384) <= wave // 2 + 1 or ch == wave
    tree = lsa.Config(k=2048, sinks=4, window=1024, mode=1)
    assert lsa.prefill_chunk(tree, 131072, 32, 8, 16384) == 16384
    assert lsa.prefill_chunk(tree, 3000, 8, 2, 700) == 700
