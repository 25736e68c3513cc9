"""Pins of the oracle's training-free PCA projection (oracle.fit_pca) against
what the mathematics fixes, independently of the function itself:

* a closed form: keys whose centred covariance is exactly diagonal (scaled
  rows of a Sylvester-Hadamard matrix) have the coordinate axes as principal
  directions, in the order of the variances;
* invariances: a shift of every key by one vector leaves the directions
  unchanged; doubling the keys multiplies the eigenvalues by 4;
* a second algorithm: the right singular vectors of the centred key matrix
  (an SVD, not an eigen-solver) span the same leading subspace, and the
  squared singular values / N are the eigenvalues;
* structure: orthonormal directions, eigenvalues in descending order,
  covariance residual ||C v - lambda v|| at rounding level, sign convention.
"""
import numpy as np
import pytest

import oracle
import synth


def _hadamard(n: int) -> np.ndarray:
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def _to_bits(x: np.ndarray) -> np.ndarray:
    b = synth.f32_to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f64(b), x), "inputs must be bf16-exact"
    return b


@pytest.mark.parametrize("hkv", [1, 2])
def test_diagonal_covariance_gives_coordinate_axes(hkv):
    d = 128
    H = _hadamard(d)                      # rows orthogonal; column 0 all ones
    dscale = 1.0 + np.arange(d) / 128.0   # distinct, bf16-exact
    X = H * dscale[None, :]               # 128 keys
    K = _to_bits(X).reshape(d // hkv, hkv, d)
    W, lam, V = oracle.fit_pca(K)
    # centred covariance = diag(dscale^2) except dim 0 (constant column: 0)
    want = np.sort(dscale[1:] ** 2)[::-1]
    assert np.allclose(lam[:d - 1], want, rtol=0, atol=1e-12)
    assert abs(lam[-1]) < 1e-12
    for j in range(64):
        e = np.zeros(d)
        e[d - 1 - j] = 1.0                # largest variance: highest dim index
        assert np.array_equal(W[:, j], e.astype(np.float32)), j


def test_shift_and_scale_invariance():
    K = synth.pca_keys(1, 512, 2)
    W, lam, _ = oracle.fit_pca(K)
    X = oracle.bf16_to_f64(K)
    # doubling is exact in bf16
    W2, lam2, _ = oracle.fit_pca(_to_bits(2.0 * X))
    assert np.allclose(lam2, 4.0 * lam, rtol=1e-12, atol=1e-12)
    assert np.allclose(W2, W, atol=1e-6)
    H = _hadamard(128) * (1.0 + np.arange(128))[None, :]   # integers up to 128
    shift = np.round(np.linspace(-3, 3, 128))               # integer sums stay below 256: bf16-exact
    Wa, la, _ = oracle.fit_pca(_to_bits(H).reshape(128, 1, 128))
    Wb, lb, _ = oracle.fit_pca(_to_bits(H + shift[None, :]).reshape(128, 1, 128))
    assert np.allclose(la, lb, atol=1e-12)
    assert np.array_equal(Wa, Wb)


def test_matches_svd_of_centred_keys():
    K = synth.pca_keys(2, 2048, 2)
    W, lam, V = oracle.fit_pca(K)
    X = oracle.bf16_to_f64(K).reshape(-1, 128)
    Xc = X - X.mean(axis=0)
    _, sv, Vt = np.linalg.svd(Xc, full_matrices=False)
    assert np.allclose(sv ** 2 / X.shape[0], lam, rtol=1e-9, atol=1e-12)
    # each leading direction agrees up to sign (spectrum well separated)
    for j in range(64):
        c = abs(float(Vt[j] @ V[:, j]))
        assert c > 1 - 1e-9, (j, c)


def test_structure():
    K = synth.pca_keys(3, 1024, 1)
    W, lam, V = oracle.fit_pca(K)
    assert W.shape == (128, 64) and W.dtype == np.float32
    assert np.all(np.diff(lam) <= 0)
    assert np.allclose(V.T @ V, np.eye(128), atol=1e-12)
    X = oracle.bf16_to_f64(K).reshape(-1, 128)
    Xc = X - X.mean(axis=0)
    C = Xc.T @ Xc / X.shape[0]
    assert np.abs(C @ V - V * lam[None, :]).max() < 1e-12 * np.abs(C).max() * 128
    # the projection holds the leading directions as its columns (fp32)
    Wd = W.astype(np.float64)
    assert np.abs(C @ Wd - Wd * lam[None, :64]).max() < 1e-5 * lam[0]
    for j in range(128):  # sign convention: the largest-magnitude entry is positive
        i = int(np.argmax(np.abs(V[:, j])))
        assert V[i, j] > 0
