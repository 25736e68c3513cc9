"""GPU parity of the sparse-attention backward (lsa_attn_backward) against
the oracle's fp64 gradients (oracle.attention_backward) on the same bf16
inputs and index rows.

Bar (derived from the arithmetic): P and dS enter the tensor-core products
rounded to bf16 (relative error 2^-9) and D = dO . O uses the bf16 forward
output, with fp32 accumulation; so every gradient is compared with
max |err| <= 2e-2 * max |ref| and mean |err| <= 2e-3 * max |ref|, the bar of
the forward attention.  An empty row gives exactly zero.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import oracle_cfg, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


def _bf16(rng, shape, scale=1.0):
    return synth.f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))


def _run(lsa, Q, K, V, dO, idx):
    """Library gradients and the oracle's, with the library's O input the
    oracle's forward output rounded to bf16."""
    O = oracle.bf16_rne(oracle.attention(Q, K, V, idx)).reshape(Q.shape)
    dQ, dK, dV = lsa.attn_backward(to_dev_bf16(Q), to_dev_bf16(K), to_dev_bf16(V), to_dev_bf16(O),
                                   to_dev_bf16(dO), to_dev(idx.astype(np.int32)))
    torch.cuda.synchronize()
    lsa.check_device_error()
    ref = oracle.attention_backward(Q, K, V, idx, dO)
    return (dQ.cpu().numpy(), dK.cpu().numpy(), dV.cpu().numpy()), ref


def _close(got, ref, what):
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got.astype(np.float64) - ref)
    assert err.max() <= 2e-2 * scale, (what, err.max() / scale)
    assert err.mean() <= 2e-3 * scale, (what, err.mean() / scale)


@pytest.mark.parametrize("hq,hkv", [(4, 1), (32, 8), (8, 8), (16, 2)])
def test_ragged_rows_match_oracle(lsa, hq, hkv):
    rng = np.random.default_rng(hq * 10 + hkv)
    nq, T, n = 37, 300, 53          # several 16-key tiles, a ragged tail
    Q, dO = _bf16(rng, (nq, hq, 128)), _bf16(rng, (nq, hq, 128))
    K, V = _bf16(rng, (T, hkv, 128)), _bf16(rng, (T, hkv, 128))
    idx = np.full((nq, hkv, n), -1, np.int32)
    for q in range(nq):
        for g in range(hkv):
            m = int(rng.integers(0, n + 1))
            idx[q, g, :m] = rng.choice(T, size=m, replace=False)
            rng.shuffle(idx[q, g])
    idx[0, 0] = -1                   # an empty row
    (dQ, dK, dV), (rQ, rK, rV) = _run(lsa, Q, K, V, dO, idx)
    G = hq // hkv
    assert np.all(dQ[0, :G] == 0)
    _close(dQ, rQ, "dQ")
    _close(dK, rK, "dK")
    _close(dV, rV, "dV")


def test_single_key_rows(lsa):
    """softmax over one key is 1 (p = 1 exactly): dV of the key is the sum of
    the group's output gradients, and dQ, dK vanish up to the rounding of
    dO . v - D (two fp32 sums of the same products in different orders)."""
    rng = np.random.default_rng(7)
    Q, dO = _bf16(rng, (3, 2, 128)), _bf16(rng, (3, 2, 128))
    K, V = _bf16(rng, (20, 1, 128)), _bf16(rng, (20, 1, 128))
    idx = np.array([[[-1, 4, -1]], [[11, -1, -1]], [[-1, -1, 17]]], np.int32)
    (dQ, dK, dV), _ = _run(lsa, Q, K, V, dO, idx)
    assert np.abs(dQ).max() <= 1e-3 and np.abs(dK).max() <= 1e-3
    dOf = oracle.bf16_to_f64(dO)
    for q, j in enumerate((4, 11, 17)):
        want = dOf[q, 0] + dOf[q, 1]
        assert np.allclose(dV[j, 0], want, rtol=2.0 ** -21, atol=1e-30)
    others = np.delete(dV, [4, 11, 17], axis=0)
    assert np.all(others == 0)


def test_lsa_rows_of_the_4k_layer(lsa):
    """Real index rows: the oracle's selection on the 4k workload at query
    positions across the sequence, gradients of the attention over them."""
    cfg = lsa.Config(k=512, sinks=4, window=256)
    inp = synth.layer_inputs("prefill-4k", seed=2)
    tpos = np.array([0, 3, 260, 777, 1500, 2048, 3000, 4095])
    r = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], oracle_cfg(cfg), tpos=tpos)
    rng = np.random.default_rng(11)
    Qs = np.ascontiguousarray(inp["Q"][tpos])
    dO = _bf16(rng, Qs.shape)
    (dQ, dK, dV), (rQ, rK, rV) = _run(lsa, Qs, inp["K"], inp["V"], dO, r["idx"])
    _close(dQ, rQ, "dQ")
    _close(dK, rK, "dK")
    _close(dV, rV, "dV")


def test_query_chunks_accumulate(lsa):
    """dK and dV are added to: two calls over the two halves of the queries
    give the gradients of one call (up to fp32 summation order)."""
    rng = np.random.default_rng(3)
    nq, hq, hkv, T, n = 40, 8, 2, 200, 32
    Q, dO = _bf16(rng, (nq, hq, 128)), _bf16(rng, (nq, hq, 128))
    K, V = _bf16(rng, (T, hkv, 128)), _bf16(rng, (T, hkv, 128))
    idx = np.stack([np.stack([rng.choice(T, size=n, replace=False) for _ in range(hkv)]) for _ in range(nq)])
    idx = idx.astype(np.int32)
    O = oracle.bf16_rne(oracle.attention(Q, K, V, idx)).reshape(Q.shape)
    dev = [to_dev_bf16(x) for x in (Q, K, V, O, dO)]
    di = to_dev(idx)
    dQa, dKa, dVa = lsa.attn_backward(*dev, di)
    h = nq // 2
    dQ1, dK2, dV2 = lsa.attn_backward(dev[0][:h], dev[1], dev[2], dev[3][:h], dev[4][:h], di[:h])
    dQ2, _, _ = lsa.attn_backward(dev[0][h:], dev[1], dev[2], dev[3][h:], dev[4][h:], di[h:], dK=dK2, dV=dV2)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([dQ1, dQ2]), dQa)
    scale = float(dKa.abs().max())
    assert float((dK2 - dKa).abs().max()) <= 1e-5 * scale
    assert float((dV2 - dVa).abs().max()) <= 1e-5 * float(dVa.abs().max())


def test_bad_arguments(lsa):
    from clustered_key_indexing_b200._lib import LSA_EINVAL, LSA_EUNSUPPORTED, LSAError
    rng = np.random.default_rng(0)
    Q = to_dev_bf16(_bf16(rng, (2, 6, 128)))
    K = to_dev_bf16(_bf16(rng, (8, 2, 128)))
    idx = to_dev(np.zeros((2, 2, 4), np.int32))
    with pytest.raises(LSAError) as e:
        lsa.attn_backward(Q, K, K, Q, Q, idx)        # hq / hkv = 3
    assert e.value.status == LSA_EUNSUPPORTED
    Q4 = to_dev_bf16(_bf16(rng, (2, 4, 128)))
    with pytest.raises(ValueError):                            # rows of 127: refused by the binding
        lsa.attn_backward(Q4[:, :, 1:], K, K, Q4, Q4, idx)
    with pytest.raises(LSAError) as e:                         # NULL dQ pointer: refused by the library
        from clustered_key_indexing_b200._lib import lib
        import ctypes
        p = ctypes.c_void_p
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        from clustered_key_indexing_b200._lib import check
        check(lib().lsa_attn_backward(p(Q4.data_ptr()), p(K.data_ptr()), p(K.data_ptr()), p(Q4.data_ptr()),
                                      p(Q4.data_ptr()), p(idx.data_ptr()), 2, 4, 2, 4, 8, None, None, None, st),
              "lsa_attn_backward")
    assert e.value.status == LSA_EINVAL
