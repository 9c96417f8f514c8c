"""Pins of the oracle's full rotation for sizes that are not a power of two
(QuaRot summary, Elamur Research, references: Sloane's library of Hadamard
matrices as the source of such factors).  The factor is Paley's first
construction over GF(p^e); the rotation is (x * diag(s)) (H_m (x) H_n) / sqrt(K).
The pins do not go through the oracle's own arithmetic: the Hadamard property
as an integer identity, Legendre symbols computed here with Python's pow,
numpy's Kronecker product, scipy's Sylvester matrix, norms and basis vectors."""
import numpy as np
import pytest
import scipy.linalg

import oracle
from rotation_bit_quantization_randomized_b200 import synth

PALEY = [(3, 1), (7, 1), (11, 1), (19, 1), (23, 1), (3, 3), (7, 3)]


@pytest.mark.parametrize("p,e", PALEY)
def test_paley_is_a_skew_hadamard_matrix(p, e):
    H = oracle.paley(p, e).astype(np.int64)
    n = p ** e + 1
    assert H.shape == (n, n)
    assert set(np.unique(H)) == {-1, 1}
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n, dtype=np.int64))
    np.testing.assert_array_equal(H + H.T, 2 * np.eye(n, dtype=np.int64))     # I + skew core
    np.testing.assert_array_equal(H[0], 1)
    np.testing.assert_array_equal(H[1:, 0], -1)


@pytest.mark.parametrize("p", [3, 7, 11, 19, 23, 31, 43])
def test_paley_prime_core_is_the_legendre_symbol_of_differences(p):
    H = oracle.paley(p, 1).astype(np.int64)
    for i in range(p):
        for j in range(p):
            if i == j:
                assert H[i + 1, j + 1] == 1
                continue
            d = (i - j) % p
            leg = pow(d, (p - 1) // 2, p)
            assert H[i + 1, j + 1] == (1 if leg == 1 else -1)


@pytest.mark.parametrize("p,e", [(3, 3), (7, 3)])
def test_paley_extension_core_depends_only_on_the_digitwise_difference(p, e):
    """Q[i][j] = chi(a_i - a_j): equal differences (digit-wise mod p) give
    equal entries, half of the nonzero differences are squares, and
    chi(-d) = -chi(d) (q = 3 mod 4)."""
    H = oracle.paley(p, e).astype(np.int64)
    q = p ** e
    digits = np.array([[(a // p ** k) % p for k in range(e)] for a in range(q)])
    weights = p ** np.arange(e)
    chi = {}
    for i in range(q):
        d = ((digits[i] - digits) % p) @ weights          # index of a_i - a_j for all j
        for j in range(q):
            if i != j:
                v = H[i + 1, j + 1]
                assert chi.setdefault(int(d[j]), v) == v
    assert len(chi) == q - 1
    assert sum(1 for v in chi.values() if v == 1) == (q - 1) // 2
    for d, v in chi.items():
        neg = int(((-digits[d]) % p) @ weights)
        assert chi[neg] == -v


@pytest.mark.parametrize("p,e,n", [(11, 1, 8), (3, 3, 4), (7, 3, 2), (3, 1, 16)])
def test_rotate_kron_equals_the_dense_kronecker_product(p, e, n):
    m = p ** e + 1
    K = m * n
    x = synth.random_f16((5, K), 31 + K, dist="student_t3")
    s = synth.signs(K, 32 + K)
    R = np.kron(oracle.paley(p, e).astype(np.float64), scipy.linalg.hadamard(n).astype(np.float64))
    ref = (x.astype(np.float64) * s) @ R / np.sqrt(K)
    got = oracle.rotate_kron(x, s, p, e)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_rotate_kron_11008_basis_vectors_norms_and_inverse():
    K, m, n = 11008, 344, 32
    H = oracle.paley(7, 3).astype(np.float64)
    Hn = scipy.linalg.hadamard(n).astype(np.float64)
    s = synth.signs(K, 40)
    # basis vectors: e_i -> s_i (H_m[a] (x) H_n[b]) / sqrt(K), i = a n + b
    idx = [0, 1, 31, 32, 5000, K - 1]
    x = np.zeros((len(idx), K), np.float16)
    for r, i in enumerate(idx):
        x[r, i] = 1.0
    got = oracle.rotate_kron(x, s)
    for r, i in enumerate(idx):
        a, b = divmod(i, n)
        np.testing.assert_allclose(got[r], s[i] * np.kron(H[a], Hn[b]) / np.sqrt(K), rtol=0, atol=1e-15)
    # an orthogonal map: norms kept, and X = H_m Y H_n^T * sqrt(K)/K undoes it
    x = synth.random_f16((3, K), 41, dist="laplace")
    y = oracle.rotate_kron(x, s)
    xs = x.astype(np.float64) * s
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(xs, axis=1), rtol=1e-13)
    back = np.stack([(H @ yr.reshape(m, n) @ Hn.T).reshape(-1) / np.sqrt(K) for yr in y])
    np.testing.assert_allclose(back, xs, rtol=0, atol=1e-12 * np.abs(xs).max())


def test_rotate_kron_spreads_an_outlier_channel():
    """One huge channel ends up spread evenly: every rotated entry of a row
    that is zero but for one channel has the same magnitude |x| / sqrt(K)."""
    K = 11008
    x = np.zeros((1, K), np.float16)
    x[0, 777] = 1000.0
    y = oracle.rotate_kron(x, np.ones(K, np.int8))
    np.testing.assert_allclose(np.abs(y), 1000.0 / np.sqrt(K), rtol=1e-15)


def test_rotate_kron_rejects_bad_sizes():
    x = np.zeros((1, 344 * 3), np.float16)
    with pytest.raises(ValueError):
        oracle.rotate_kron(x, np.ones(344 * 3, np.int8))          # 3 is not a power of two
    with pytest.raises(ValueError):
        oracle.paley(5, 1)                                       # 5 = 1 mod 4
    with pytest.raises(ValueError):
        oracle.paley(9, 1)                                       # 9 is not a prime


def test_rotate_quant_kron_composes_rotation_and_rtn():
    K = 11008
    x = synth.random_f16((4, K), 43, dist="laplace")
    s = synth.signs(K, 43)
    packed, sc, xr = oracle.rotate_quant_kron(x, s, group=128)
    codes = oracle.unpack(packed)
    step = oracle.f16_to_f64(sc).repeat(128, axis=1)
    assert np.all(np.abs(xr - step * codes) <= step / 2 * (1 + 1e-12) + 1e-300)
    packed0, sc0, _ = oracle.rotate_quant_kron(x, s, group=0)
    np.testing.assert_allclose(sc0, np.abs(xr).max(axis=1) / 7, rtol=1e-15)
