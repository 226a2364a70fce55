"""Pins of the oracle's Walsh-Hadamard rotation and of the paired-transform
invariant (Dual-QK summary, Sec. 1 and Sec. 3.1: the query transform and the
inverse-transpose key transform preserve q.k before quantization; the
Hadamard rotation is the orthonormal special case T^{-T} = T).
"""
import numpy as np
import pytest

from oracle import oracle as orc


def sylvester(d):
    """Dense Hadamard matrix from its definition H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(d)[:, None]
    j = np.arange(d)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1.0, -1.0)


@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_matches_dense_definition(d):
    rng = np.random.default_rng(d)
    H = sylvester(d)
    for _ in range(5):
        x = rng.integers(-1000, 1000, size=d).astype(np.float64)  # integer inputs: every sum exact
        np.testing.assert_array_equal(orc.fwht(x), H @ x)


def test_rotate_basis_vectors_give_rows_of_normalized_h():
    d = 128
    H = sylvester(d) / np.sqrt(d)
    for i in [0, 1, 5, 64, 127]:
        e = np.zeros(d, np.float32)
        e[i] = 1.0
        np.testing.assert_array_equal(orc.rotate(e), H[i].astype(np.float32))


def test_fwht_involution_and_parseval():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(128)
    y = orc.fwht(x)
    np.testing.assert_allclose(orc.fwht(y), 128 * x, rtol=0, atol=1e-12)
    assert abs(np.dot(y, y) / 128 - np.dot(x, x)) <= 1e-12 * np.dot(x, x)


def test_rotation_preserves_dot_products_before_quantization():
    rng = np.random.default_rng(2)
    for _ in range(20):
        q = rng.standard_normal(128)
        k = rng.standard_normal(128) * np.exp(0.5 * rng.standard_normal(128))
        qr, kr = orc.fwht(q) / np.sqrt(128), orc.fwht(k) / np.sqrt(128)
        assert abs(qr @ kr - q @ k) <= 1e-12 * np.abs(q) @ np.abs(k)
        # the fp32-rounded rotation keeps it to fp32 accuracy
        q32, k32 = q.astype(np.float32), k.astype(np.float32)
        r = orc.rotate(q32).astype(np.float64) @ orc.rotate(k32).astype(np.float64)
        assert abs(r - q32.astype(np.float64) @ k32.astype(np.float64)) <= 1e-6 * np.abs(q) @ np.abs(k)


def test_dual_transform_pair_preserves_scores():
    rng = np.random.default_rng(3)
    d = 32
    for _ in range(10):
        U, _ = np.linalg.qr(rng.standard_normal((d, d)))
        V, _ = np.linalg.qr(rng.standard_normal((d, d)))
        T = U @ np.diag(np.exp(rng.uniform(-1.5, 1.5, d))) @ V  # non-orthogonal, cond <= e^3
        q, k = rng.standard_normal(d), rng.standard_normal(d)
        cond = np.linalg.cond(T)
        assert abs(orc.dual_score(T, q, k) - q @ k) <= cond * 1e-13 * np.abs(q) @ np.abs(k) * d


def test_hadamard_is_the_self_inverse_transpose_special_case():
    d = 64
    T = sylvester(d) / np.sqrt(d)
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    # T^{-T} = T for the orthonormal Hadamard, so the pair is FWHT on both sides
    ref = (orc.fwht(q) / np.sqrt(d)) @ (orc.fwht(k) / np.sqrt(d))
    assert abs(orc.dual_score(T, q, k) - ref) <= 1e-12 * np.abs(q) @ np.abs(k)


def test_dual_score_rejects_singular_transform():
    T = np.eye(8)
    T[3, :] = T[2, :]
    assert np.isnan(orc.dual_score(T, np.ones(8), np.ones(8)))
