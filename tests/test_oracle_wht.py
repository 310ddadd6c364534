"""Pins of the oracle's Walsh-Hadamard rotation (Bonsai-Ternary-27B page, section
"How the Walsh-Hadamard transform and Sinkhorn save quality at 4-bit": the rotation mixes
each head vector).  Closed form: the Sylvester matrix H_ij = (-1)^popcount(i & j)."""
from decimal import Decimal, getcontext

import numpy as np

import oracle

D = 128


def sylvester():
    i = np.arange(D)
    pc = np.vectorize(lambda x: bin(int(x)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


def kappa():
    return np.float32(oracle.wht128(np.eye(D, dtype=np.float32)[0])[0])


def test_kappa_is_nearest_fp32_to_2_pow_minus_3_5():
    getcontext().prec = 60
    exact = Decimal(2) ** Decimal(-3.5)
    k = kappa()
    nb = [np.nextafter(k, np.float32(0)), k, np.nextafter(k, np.float32(1))]
    errs = [abs(Decimal(float(v)) - exact) for v in nb]
    assert errs[1] < errs[0] and errs[1] < errs[2]


def test_basis_vectors_give_sylvester_columns():
    H = sylvester()
    k = kappa()
    cols = oracle.wht128(np.eye(D, dtype=np.float32))  # row r = transform of e_r
    ints = cols / k
    assert np.array_equal(ints, np.rint(ints))  # exact: integer arithmetic before kappa
    assert np.array_equal(ints.astype(np.int64).T, H)


def test_orthogonality_in_integers():
    k = kappa()
    H = (oracle.wht128(np.eye(D, dtype=np.float32)) / k).astype(np.int64)
    assert np.array_equal(H @ H.T, 128 * np.eye(D, dtype=np.int64))


def test_rotate_twice_recovers_input():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((64, D)) * np.exp2(rng.integers(-4, 5, (64, 1)))).astype(np.float32)
    x2 = oracle.wht128(oracle.wht128(x))
    # kappa^2 * 128 = 1 - 3.4e-8; each of the 14 butterfly stages rounds once per element
    bound = 2.0**-17 * np.abs(x).max(axis=1, keepdims=True)
    assert np.all(np.abs(x2 - x) <= bound)


def test_matches_fp64_matrix_product():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((32, D)).astype(np.float32)
    ref = (x.astype(np.float64) @ sylvester().T.astype(np.float64)) * float(kappa())
    got = oracle.wht128(x).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0**-19 * np.abs(x).sum(axis=1, keepdims=True))


def test_fp64_rotation_is_orthonormal_inverse():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, D))
    y = oracle.wht128_f64(oracle.wht128_f64(x))
    assert np.allclose(y, x, atol=1e-13)
    ref = x @ sylvester().T / np.sqrt(128.0)
    assert np.allclose(oracle.wht128_f64(x), ref, atol=1e-13)
