"""The Python binding refuses, before any library call, arguments whose dtype
or shape differs from the dense layout the library reads (bf16 [*, *, 128]
Q/K/V, fp32 [128, 64] projections, int32 index rows of the documented
shape).  A wrong layout would otherwise be read as if it were the right one,
possibly past the end of the tensor.  No GPU needed: the checks run first,
and a well-formed CPU tensor then stops at the CUDA check."""
import types

import pytest
import torch

import clustered_key_indexing_b200 as lsa
from clustered_key_indexing_b200 import _lib

bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def z(*shape, dtype=bf16):
    return torch.zeros(shape, dtype=dtype)


W = z(128, 64, dtype=f32)


def test_build_and_latent_checks():
    cfg = lsa.Config()
    cache = types.SimpleNamespace(hkv=2)
    with pytest.raises(TypeError, match="K: expected torch.bfloat16"):
        lsa.build_buckets(z(16, 2, 128, dtype=f32), W, cfg, cache)
    with pytest.raises(ValueError, match="K: expected shape"):
        lsa.build_buckets(z(16, 2, 64), W, cfg, cache)
    with pytest.raises(ValueError, match="W_k: expected shape"):
        lsa.build_buckets(z(16, 2, 128), z(64, 64, dtype=f32), cfg, cache)
    with pytest.raises(ValueError, match="CUDA tensors"):
        lsa.build_buckets(z(16, 2, 128), W, cfg, cache)
    with pytest.raises(TypeError, match="W_q"):
        lsa.query_latent(z(4, 8, 128), z(128, 64, dtype=torch.float64), 2, cfg)
    with pytest.raises(ValueError, match="K: expected shape"):
        lsa.fit_pca(z(16, 2, 127))


def test_select_and_attention_checks():
    cfg = lsa.Config(k=64, sinks=4, window=32)
    cache = types.SimpleNamespace(hkv=2)
    Q = z(5, 8, 128)
    with pytest.raises(ValueError, match="idx: expected shape"):
        lsa.select(Q, 0, W, cache, cfg, idx=z(5, 2, cfg.row + 1, dtype=i32))
    with pytest.raises(TypeError, match="idx: expected torch.int32"):
        lsa.select(Q, 0, W, cache, cfg, idx=z(5, 2, cfg.row, dtype=torch.int64))
    with pytest.raises(ValueError, match="Y_out: expected shape"):
        lsa.select(Q, 0, W, cache, cfg, Y_out=z(5, 8, 64))          # mean variant: one row per kv-head
    with pytest.raises(ValueError, match="CUDA tensors"):
        lsa.select(Q, 0, W, cache, cfg, idx=z(5, 2, cfg.row, dtype=i32), Y_out=z(5, 2, 64))
    K = z(100, 2, 128)
    with pytest.raises(ValueError, match="V: expected shape"):
        lsa.sparse_attn(Q, K, z(99, 2, 128), z(5, 2, 7, dtype=i32))
    with pytest.raises(ValueError, match="idx: expected shape"):
        lsa.sparse_attn(Q, K, K, z(5, 4, 7, dtype=i32))
    with pytest.raises(ValueError, match="O: expected shape"):
        lsa.sparse_attn(Q, K, K, z(5, 2, 7, dtype=i32), O=z(5, 8, 64))
    with pytest.raises(ValueError, match="idx: expected shape"):
        lsa.select_attn(Q, K, K, z(5, 2, 7, dtype=i32), 0, cfg)        # rows of S + k + W
    with pytest.raises(ValueError, match="CUDA tensors"):
        lsa.select_attn(Q, K, K, z(5, 2, cfg.row, dtype=i32), 0, cfg)


def test_prefill_checks():
    cfg = lsa.Config()
    Q, K = z(64, 8, 128), z(64, 2, 128)
    with pytest.raises(ValueError, match="K: expected shape"):
        lsa.prefill(Q, z(63, 2, 128), z(63, 2, 128), W, W, cfg)
    with pytest.raises(ValueError, match="O: expected shape"):
        lsa.prefill(Q, K, K, W, W, cfg, O=z(64, 8, 64))
    with pytest.raises(ValueError, match="hV: expected shape"):
        lsa.prefill_host(Q, K, z(64, 1, 128), W, W, cfg)
    with pytest.raises(ValueError, match="Q: expected shape"):
        lsa.prefill_host(Q, K, K, W, W, cfg, dev_bufs=(z(64, 8, 64), K, K, Q))


def test_decode_checks():
    dec = lsa.Decode.__new__(lsa.Decode)     # the state's shape only; nothing allocated
    dec.d = _lib.lsa_decode()
    dec.d.batch, dec.d.hkv, dec.d.hq = 3, 2, 8
    dec.cfg = lsa.Config(k=64, sinks=4, window=32)
    dec.K = z(3, 512, 2, 128)
    q, kv = z(3, 8, 128), z(3, 2, 128)
    with pytest.raises(ValueError, match="q: expected shape"):
        dec.step(z(2, 8, 128), kv, kv, W, W)
    with pytest.raises(ValueError, match="v: expected shape"):
        dec.step(q, kv, z(3, 1, 128), W, W)
    with pytest.raises(ValueError, match="idx_out: expected shape"):
        dec.step(q, kv, kv, W, W, idx_out=z(3, 2, 5, dtype=i32))
    with pytest.raises(ValueError, match="CUDA tensors"):
        dec.step(q, kv, kv, W, W, idx_out=z(3, 2, dec.cfg.row, dtype=i32))
    with pytest.raises(ValueError, match="K: expected shape"):
        dec.load(0, z(40, 3, 128), z(40, 3, 128), W)
