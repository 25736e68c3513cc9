"""Pins of the oracle's sparse-attention backward (oracle.attention_backward):
the gradients of exact softmax attention over saved index lists (tutorial
"隐空间稀疏注意力 (LSA)", section 二, for the attention; essay "《卡片柜》",
ch. 6: the natively trained variant keeps the selected key indices of every
query for its backward pass).

Independent checks:
* a library routine: torch autograd of scaled_dot_product_attention (fp64)
  when every list is the full causal prefix, with 8 kv-heads of 4 query heads;
* a library routine: torch autograd of a gathered, masked softmax on ragged
  lists (padding, an empty list, single-key lists, different lists per head);
* central finite differences of sum(dO * O), O from a forward written here;
* closed forms and invariants: single-key and empty lists; the key gradients
  of one kv-head sum to zero (a shift of every key leaves each softmax
  unchanged); the value gradients sum to the output gradients; dV does not
  depend on V, and dQ, dK are linear in V.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _rng(seed):
    return np.random.default_rng(seed)


def _ref_gather(Q, K, V, idx, dO):
    """torch autograd of attention over index lists, written with gather and a
    masked softmax (fp64)."""
    Q = torch.tensor(Q, requires_grad=True)
    K = torch.tensor(K, requires_grad=True)
    V = torch.tensor(V, requires_grad=True)
    nq, hq, d = Q.shape
    hkv = K.shape[1]
    G = hq // hkv
    ix = torch.tensor(idx.astype(np.int64))                 # [nq, hkv, n]
    valid = ix >= 0
    safe = ix.clamp(min=0)
    heads = torch.arange(hkv)[None, :, None].expand_as(safe)
    Kg = K[safe, heads]                                     # [nq, hkv, n, d]
    Vg = V[safe, heads]
    Kg = Kg.repeat_interleave(G, dim=1)                     # [nq, hq, n, d]
    Vg = Vg.repeat_interleave(G, dim=1)
    m = valid.repeat_interleave(G, dim=1)
    s = torch.einsum("qhd,qhnd->qhn", Q, Kg) / np.sqrt(d)
    s = s.masked_fill(~m, float("-inf"))
    p = torch.softmax(s, dim=-1)
    p = torch.nan_to_num(p, nan=0.0)                        # empty lists
    O = torch.einsum("qhn,qhnd->qhd", p, Vg)
    (O * torch.tensor(dO)).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def _forward(Q, K, V, idx):
    """fp64 sparse attention written as plain loops (for finite differences)."""
    nq, hq, d = Q.shape
    G = hq // K.shape[1]
    O = np.zeros_like(Q)
    for q in range(nq):
        for h in range(hq):
            keys = [j for j in idx[q, h // G] if j >= 0]
            if not keys:
                continue
            s = np.array([Q[q, h] @ K[j, h // G] for j in keys]) / np.sqrt(d)
            w = np.exp(s - s.max())
            w /= w.sum()
            O[q, h] = sum(wi * V[j, h // G] for wi, j in zip(w, keys))
    return O


def _ragged_lists(rng, nq, hkv, n, T):
    idx = np.full((nq, hkv, n), -1, np.int32)
    for q in range(nq):
        for g in range(hkv):
            m = int(rng.integers(0, n + 1))
            idx[q, g, :m] = rng.choice(T, size=m, replace=False)
            rng.shuffle(idx[q, g])                          # padding anywhere
    idx[0, 0] = -1                                          # an empty list
    idx[1, 0] = -1
    idx[1, 0, 2] = T - 1                                    # a single key
    return idx


def test_full_causal_gradients_match_sdpa_autograd():
    T = 64
    rng = _rng(1)
    # bf16 inputs of the 8 kv-head / 32 query-head geometry
    Qb, Kb, Vb = (synth.f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
                  for s in ((T, 32, 128), (T, 8, 128), (T, 8, 128)))
    Q, K, V = (oracle.bf16_to_f64(x) for x in (Qb, Kb, Vb))
    dO = rng.standard_normal(Q.shape)
    idx = np.full((T, 8, T), -1, np.int32)
    for t in range(T):
        idx[t, :, :t + 1] = np.arange(t + 1)
    dQ, dK, dV = oracle.attention_backward(Qb, Kb, Vb, idx, dO)
    q = torch.tensor(Q).permute(1, 0, 2).requires_grad_()
    k = torch.tensor(K).permute(1, 0, 2).requires_grad_()
    v = torch.tensor(V).permute(1, 0, 2).requires_grad_()
    O = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(4, dim=0), v.repeat_interleave(4, dim=0), is_causal=True)
    (O * torch.tensor(dO).permute(1, 0, 2)).sum().backward()
    for got, ref in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
        ref = ref.permute(1, 0, 2).numpy()
        assert np.allclose(got, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))


@pytest.mark.parametrize("seed", range(3))
def test_ragged_lists_match_autograd(seed):
    rng = _rng(10 + seed)
    nq, hq, hkv, d, T, n = 5, 6, 3, 32, 40, 12
    Q = rng.standard_normal((nq, hq, d))
    K = rng.standard_normal((T, hkv, d))
    V = rng.standard_normal((T, hkv, d))
    dO = rng.standard_normal((nq, hq, d))
    idx = _ragged_lists(rng, nq, hkv, n, T)
    got = oracle.attention_backward(Q, K, V, idx, dO)
    ref = _ref_gather(Q, K, V, idx, dO)
    for a, b in zip(got, ref):
        assert np.allclose(a, b, rtol=0, atol=1e-13 * max(1.0, np.abs(b).max()))


def test_finite_differences():
    rng = _rng(3)
    nq, hq, hkv, d, T = 2, 4, 2, 4, 7
    Q = rng.standard_normal((nq, hq, d))
    K = rng.standard_normal((T, hkv, d))
    V = rng.standard_normal((T, hkv, d))
    dO = rng.standard_normal((nq, hq, d))
    idx = np.array([[[0, 3, -1, 6], [2, -1, 5, 1]],
                    [[4, 1, 2, -1], [6, 0, -1, -1]]], np.int32)
    grads = oracle.attention_backward(Q, K, V, idx, dO)
    eps = 1e-5
    for which, X in enumerate((Q, K, V)):
        num = np.zeros_like(X)
        for pos in np.ndindex(X.shape):
            args = [Q, K, V]
            Xp, Xm = X.copy(), X.copy()
            Xp[pos] += eps
            Xm[pos] -= eps
            args[which] = Xp
            fp = (_forward(*args, idx) * dO).sum()
            args[which] = Xm
            fm = (_forward(*args, idx) * dO).sum()
            num[pos] = (fp - fm) / (2 * eps)
        assert np.allclose(grads[which], num, rtol=0, atol=1e-8), which


def test_closed_forms_and_invariants():
    rng = _rng(4)
    nq, hq, hkv, d, T, n = 6, 8, 2, 16, 30, 10
    Q = rng.standard_normal((nq, hq, d))
    K = rng.standard_normal((T, hkv, d))
    V = rng.standard_normal((T, hkv, d))
    dO = rng.standard_normal((nq, hq, d))
    idx = _ragged_lists(rng, nq, hkv, n, T)
    dQ, dK, dV = oracle.attention_backward(Q, K, V, idx, dO)
    G = hq // hkv
    # query 0 / kv-head 0: empty list, no gradient; query 1 / kv-head 0: one key
    assert np.all(dQ[0, :G] == 0)
    assert np.all(dQ[1, :G] == 0)
    # a shift of every key leaves each softmax unchanged
    scale = np.abs(dK).max()
    assert np.abs(dK.sum(axis=0)).max() <= 1e-13 * scale * T
    # value gradients add up to the output gradients of the non-empty lists
    want = np.zeros((hkv, d))
    for q in range(nq):
        for h in range(hq):
            if (idx[q, h // G] >= 0).any():
                want[h // G] += dO[q, h]
    assert np.allclose(dV.sum(axis=0), want, rtol=0, atol=1e-12)
    # dV does not depend on V; dQ, dK are linear in V; all are linear in dO
    dQ2, dK2, dV2 = oracle.attention_backward(Q, K, 2.0 * V, idx, dO)
    assert np.array_equal(dV2, dV)
    assert np.allclose(dQ2, 2.0 * dQ, rtol=0, atol=1e-13 * np.abs(dQ).max())
    assert np.allclose(dK2, 2.0 * dK, rtol=0, atol=1e-13 * np.abs(dK).max())
    dQ3, dK3, dV3 = oracle.attention_backward(Q, K, V, idx, 0.5 * dO)
    assert np.array_equal(dQ3, 0.5 * dQ) and np.array_equal(dV3, 0.5 * dV)


def test_single_key_list_closed_form():
    """softmax over one key is 1 whatever the logit: dQ = 0 and dK = 0 for
    that key, and dV of the key is the output gradient."""
    rng = _rng(6)
    Q = rng.standard_normal((1, 2, 8))
    K = rng.standard_normal((5, 1, 8))
    V = rng.standard_normal((5, 1, 8))
    dO = rng.standard_normal((1, 2, 8))
    idx = np.array([[[-1, 3, -1]]], np.int32)
    dQ, dK, dV = oracle.attention_backward(Q, K, V, idx, dO)
    assert np.all(dQ == 0) and np.all(dK == 0)
    assert np.array_equal(dV[3, 0], dO[0, 0] + dO[0, 1])
    assert np.all(np.delete(dV, 3, axis=0) == 0)
