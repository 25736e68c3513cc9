"""Pins for the oracle's numeric building blocks: bf16 rounding and the
key / query latents (essay "《卡片柜》", ch. 2; tutorial "隐空间稀疏注意力",
section 二).  Each check compares with something other than the oracle itself:
brute force over all bf16 values, closed forms, or invariances."""
import math

import numpy as np
import pytest

import oracle
import synth


def _all_bf16_sorted():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)  # non-negative finite values
    vals = oracle.bf16_to_f64(bits)
    return bits, vals


def _nearest_bf16_bruteforce(x):
    """Nearest non-negative finite bf16 by exhaustive search, ties to even."""
    bits, vals = _all_bf16_sorted()
    out = []
    for v in np.abs(x):
        i = np.searchsorted(vals, v)
        cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
        best = min(cands, key=lambda j: (abs(vals[j] - v), int(bits[j]) & 1))
        if v > vals[-1] + (vals[-1] - vals[-2]) / 2 or (v == vals[-1] + (vals[-1] - vals[-2]) / 2):
            out.append(0x7F80)
        else:
            out.append(int(bits[best]))
    sign = np.where(np.signbit(x), 0x8000, 0)
    return (np.array(out, np.uint32) | sign.astype(np.uint32)).astype(np.uint16)


def test_bf16_rne_matches_bruteforce_nearest():
    rng = np.random.default_rng(1)
    bits, vals = _all_bf16_sorted()
    # exact values, midpoints, and points just off the midpoints
    pick = rng.integers(1, len(vals) - 1, 400)
    mids = (vals[pick] + vals[pick + 1]) / 2
    x = np.concatenate([
        vals[pick], mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf),
        rng.standard_normal(400) * 10.0 ** rng.integers(-30, 30, 400),
        -rng.random(200), [0.0, 1.0, -1.0, 0.5, 3.0e38, 3.4e38, 1e-39, 9.2e-41],
    ])
    got = oracle.bf16_rne(x)
    want = _nearest_bf16_bruteforce(x)
    assert np.array_equal(got, want)


def test_bf16_rne_special_values():
    assert oracle.bf16_rne(np.array([np.inf]))[0] == 0x7F80
    assert oracle.bf16_rne(np.array([-np.inf]))[0] == 0xFF80
    assert oracle.bf16_rne(np.array([np.nan]))[0] == 0x7FC0
    assert oracle.bf16_rne(np.array([-0.0]))[0] == 0x8000
    # 1 + 2^-8 is the midpoint between 1 and 1 + 2^-7: ties to even -> 1.0
    assert oracle.bf16_rne(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    # 1 + 3*2^-8 is the midpoint between 1+2^-7 (odd) and 1+2^-6 (even)
    assert oracle.bf16_rne(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82


def _identity_projection(d=128, dl=64):
    W = np.zeros((d, dl), np.float32)
    W[np.arange(dl), np.arange(dl)] = 1.0
    return W


def test_key_latent_closed_form_identity_projection():
    """W_k = [I; 0] reduces the latent to the normalised first dl coordinates."""
    rng = np.random.default_rng(2)
    K = synth.f32_to_bf16_bits(rng.standard_normal((37, 2, 128)).astype(np.float32))
    U = oracle.key_latent_pool(K, _identity_projection(), pool=1)
    Kf = oracle.bf16_to_f64(K)[:, :, :64]
    want = Kf / np.linalg.norm(Kf, axis=2, keepdims=True)
    assert np.allclose(U.transpose(1, 0, 2), want, atol=1e-15, rtol=0)


def test_key_latent_unit_norm_and_scale_invariance():
    rng = np.random.default_rng(3)
    K = synth.f32_to_bf16_bits(rng.standard_normal((64, 3, 128)).astype(np.float32))
    W = synth.orthonormal(5, "wk", 128, 64)
    Z = oracle.key_latent_pool(K, W, pool=1)
    assert np.allclose(np.linalg.norm(Z, axis=2), 1.0, atol=1e-14)
    # doubling a key is exact in bf16 and must not move its latent
    K2 = synth.f32_to_bf16_bits(2.0 * synth.bf16_bits_to_f32(K))
    Z2 = oracle.key_latent_pool(K2, W, pool=1)
    assert np.array_equal(Z, Z2)
    # a zero key has a zero latent
    Kz = K.copy()
    Kz[5, 1] = 0
    Zz = oracle.key_latent_pool(Kz, W, pool=1)
    assert np.all(Zz[1, 5] == 0.0)


def test_pooling_is_mean_of_per_key_latents_with_ragged_tail():
    rng = np.random.default_rng(4)
    T = 4 * 9 + 3  # ragged last unit of 3 keys
    K = synth.f32_to_bf16_bits(rng.standard_normal((T, 2, 128)).astype(np.float32))
    W = synth.orthonormal(6, "wk", 128, 64)
    Z = oracle.key_latent_pool(K, W, pool=1)
    U = oracle.key_latent_pool(K, W, pool=4)
    assert U.shape == (2, 10, 64)
    for j in range(10):
        want = Z[:, 4 * j:min(4 * j + 4, T)].mean(axis=1)
        assert np.allclose(U[:, j], want, atol=1e-15, rtol=0)
    # four identical keys pool to that key's (unit-norm) latent
    K[8:12] = K[8]
    U = oracle.key_latent_pool(K, W, pool=4)
    assert np.allclose(np.linalg.norm(U[:, 2], axis=1), 1.0, atol=1e-14)


def test_query_latent_closed_form_and_group_mean():
    rng = np.random.default_rng(7)
    Q = synth.f32_to_bf16_bits(rng.standard_normal((11, 8, 128)).astype(np.float32))
    W = _identity_projection()
    Qf = oracle.bf16_to_f64(Q)[:, :, :64]
    z = Qf / np.linalg.norm(Qf, axis=2, keepdims=True)
    Yn = oracle.query_latent(Q, W, hkv=2, agg=1)
    assert Yn.shape == (11, 8, 64)
    assert np.array_equal(Yn, oracle.bf16_rne(z.reshape(-1)).reshape(z.shape))
    Ym = oracle.query_latent(Q, W, hkv=2, agg=0)
    assert Ym.shape == (11, 2, 64)
    zm = z.reshape(11, 2, 4, 64).mean(axis=2)
    # the group mean is rounded once; fp64 summation order can differ only by
    # an ulp, which moves a bf16 rounding only at an exact midpoint
    assert np.mean(Ym == oracle.bf16_rne(zm.reshape(-1)).reshape(zm.shape)) > 0.999


def test_bf16_dot_exact_in_any_order_when_exponent_spread_is_small():
    """The lemma behind the tree descent's parallel exact scores: with bf16
    factors (8-bit significands) and nonzero-exponent spreads summing to at
    most 30 over the two vectors, every fp64 partial sum is exact, so any
    summation order equals the ascending sequential fma chain."""
    import random
    rng = np.random.default_rng(5)

    def bf16_vec(lo_exp, hi_exp):
        e = rng.integers(lo_exp, hi_exp + 1, size=64)
        m = rng.integers(128, 256, size=64)
        s = rng.choice([-1.0, 1.0], size=64)
        return s * m * np.exp2(e - 7.0)

    def seq(y, c):
        acc = 0.0
        for a, b in zip(y, c):
            acc = acc + a * b  # each product is exact in fp64
        return acc

    for _ in range(200):
        y = bf16_vec(-12, 0)     # spread 12
        c = bf16_vec(-18, 0)     # spread 18: total 30
        ref = seq(y, c)
        prods = list(y * c)
        for _ in range(5):
            random.shuffle(prods)
            assert sum(prods) == ref
            assert math.fsum(prods) == ref
    # and the bound is needed: widely spread exponents lose the exactness
    y = np.array([1.0, 2.0 ** -60, -1.0] + [0.0] * 61)
    c = np.ones(64)
    assert seq(y, c) != math.fsum(list(y * c))
