"""Pins for the CPU oracle: each check compares it with something it does not
compute itself (numpy's Kronecker product and matrix product, torch's batched
matmul, closed forms, hand-worked fixtures under tests/golden/).

Source of the definition: the taxoreview.com page on Kronecker-sparse matrix
multiplication, first abstract (supports are Kronecker products of identity
and all-ones blocks; butterfly/Monarch matrices are products of KS factors),
read with the textbook Kronecker index order.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = [p for p in itertools.product((1, 2, 3), repeat=4)] + [
    (4, 1, 3, 2), (1, 4, 4, 1), (2, 4, 4, 2), (3, 2, 4, 1), (1, 3, 2, 4), (4, 4, 4, 4)]


def rng(seed=0):
    return np.random.default_rng(seed)


def kron_dense(values, pattern):
    """K built only from numpy's Kronecker product: sum over (i, l) of
    E_a(i) (x) V[i, l] (x) E_d(l), E(i) the unit matrix with a one at (i, i)."""
    a, b, c, d = pattern
    V = np.asarray(values, dtype=np.float64).reshape(a, d, b, c)
    K = np.zeros((a * b * d, a * c * d))
    for i in range(a):
        Ei = np.zeros((a, a))
        Ei[i, i] = 1.0
        for l in range(d):
            El = np.zeros((d, d))
            El[l, l] = 1.0
            K += np.kron(np.kron(Ei, V[i, l]), El)
    return K


def rand_case(pattern, n=5, seed=0):
    a, b, c, d = pattern
    r = rng(seed)
    X = r.standard_normal((n, a * c * d))
    V = r.standard_normal((a, d, b, c))
    return X, V


@pytest.mark.parametrize("pattern", TINY)
def test_brute_force_against_kron(pattern):
    X, V = rand_case(pattern, seed=sum(pattern))
    K = kron_dense(V, pattern)
    np.testing.assert_array_equal(oracle.densify(V, pattern), K)
    np.testing.assert_allclose(oracle.matmul(X, V, pattern), X @ K.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pattern", [(1, 1, 1, 1), (2, 3, 4, 1), (3, 2, 2, 3), (2, 4, 4, 2), (4, 2, 3, 5)])
def test_support_is_identity_ones_identity(pattern):
    a, b, c, d = pattern
    S = np.kron(np.kron(np.eye(a), np.ones((b, c))), np.eye(d))
    np.testing.assert_array_equal(oracle.densify(np.ones(a * b * c * d), pattern), S)
    _, V = rand_case(pattern)  # standard normal: nonzero with probability one
    K = oracle.densify(V, pattern)
    assert np.count_nonzero(K) == a * b * c * d
    assert np.array_equal(K != 0, S != 0)


@pytest.mark.parametrize("b,c", [(1, 1), (3, 5), (8, 2), (16, 16)])
def test_a_d_one_is_dense_gemm(b, c):
    X, V = rand_case((1, b, c, 1), n=7)
    np.testing.assert_allclose(oracle.matmul(X, V, (1, b, c, 1)), X @ V[0, 0].T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("a,d", [(1, 1), (3, 1), (1, 4), (5, 3)])
def test_b_c_one_is_diagonal_scaling(a, d):
    X, V = rand_case((a, 1, 1, d), n=6)
    # feature f = i*d + l is scaled by values[i, l, 0, 0]
    np.testing.assert_array_equal(oracle.matmul(X, V, (a, 1, 1, d)), X * V.reshape(1, a * d))


@pytest.mark.parametrize("pattern", [(3, 4, 2, 1), (2, 5, 3, 1)])
def test_d_one_is_block_diagonal(pattern):
    a, b, c, _ = pattern
    X, V = rand_case(pattern)
    Y = oracle.matmul(X, V, pattern)
    for i in range(a):
        np.testing.assert_allclose(Y[:, i * b:(i + 1) * b], X[:, i * c:(i + 1) * c] @ V[i, 0].T,
                                   rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pattern", [(1, 3, 4, 2), (1, 2, 5, 4)])
def test_a_one_is_stride_d_interleave(pattern):
    _, b, c, d = pattern
    X, V = rand_case(pattern)
    Y = oracle.matmul(X, V, pattern).reshape(-1, b, d)
    Xr = X.reshape(-1, c, d)
    for l in range(d):
        np.testing.assert_allclose(Y[:, :, l], Xr[:, :, l] @ V[0, l].T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pattern", [(2, 4, 4, 2), (3, 2, 5, 4), (1, 6, 3, 7)])
def test_permute_bmm_identity(pattern):
    """K = P_out * blockdiag(V[i,l]) * P_in^T: permute, batched matmul, permute
    back, with torch's CPU bmm as an independent second computation."""
    a, b, c, d = pattern
    X, V = rand_case(pattern, n=9)
    Xt = torch.from_numpy(X).reshape(9, a, c, d).permute(1, 3, 0, 2).reshape(a * d, 9, c)
    Vt = torch.from_numpy(V).reshape(a * d, b, c)
    Yt = torch.bmm(Xt, Vt.transpose(1, 2)).reshape(a, d, 9, b).permute(2, 0, 3, 1).reshape(9, a * b * d)
    np.testing.assert_allclose(oracle.matmul(X, V, pattern), Yt.numpy(), rtol=1e-12, atol=1e-12)


def test_dense_matmul_is_numpy_product():
    r = rng(3)
    X, K = r.standard_normal((4, 7)), r.standard_normal((5, 7))
    np.testing.assert_allclose(oracle.dense_matmul(X, K), X @ K.T, rtol=1e-12, atol=1e-12)


CHAINS = [
    [(1, 2, 2, 4), (2, 2, 2, 2), (4, 2, 2, 1)],        # butterfly, size 8
    [(4, 4, 4, 1), (1, 4, 4, 4)],                      # Monarch-like, size 16
    [(2, 3, 2, 1), (1, 2, 3, 2), (1, 3, 4, 1)],        # rectangular widths 4 -> 6 -> 4 -> 3
]


@pytest.mark.parametrize("patterns", CHAINS)
def test_chain_is_densified_product(patterns):
    r = rng(11)
    a0, b0, c0, d0 = patterns[0]
    X = r.standard_normal((5, a0 * c0 * d0))
    facs = [r.standard_normal(a * b * c * d) for (a, b, c, d) in patterns]
    M = np.eye(a0 * c0 * d0)
    for V, p in zip(facs, patterns):
        M = kron_dense(V, p) @ M
    np.testing.assert_allclose(oracle.chain(X, facs, patterns), X @ M.T, rtol=1e-11, atol=1e-11)


def test_chain_rejects_width_mismatch():
    with pytest.raises(ValueError):
        oracle.chain(np.zeros((1, 4)), [np.zeros(8), np.zeros(8)], [(1, 2, 2, 2), (1, 2, 2, 1)])


def hadamard_values(pattern):
    a, b, c, d = pattern
    # every 2x2 block equals H_2: values[i, l, k, j] = (-1)^(k*j)
    blk = np.array([[1.0, 1.0], [1.0, -1.0]])
    return np.broadcast_to(blk, (a, d, b, c)).copy()


@pytest.mark.parametrize("m", [1, 3, 6])
def test_butterfly_of_h2_blocks_is_sylvester_hadamard(m):
    n = 2 ** m
    pats = [(2 ** (k - 1), 2, 2, 2 ** (m - k)) for k in range(1, m + 1)]
    H = oracle.chain(np.eye(n), [hadamard_values(p) for p in pats], pats)
    r = np.arange(n)
    closed = np.array([[(-1.0) ** bin(x & y).count("1") for y in r] for x in r])
    np.testing.assert_array_equal(H, closed)  # I * H^T, and H is symmetric


def test_golden_sylvester_hadamard_8():
    H8 = np.loadtxt(os.path.join(GOLDEN, "sylvester_hadamard_8.txt"))
    pats = [(1, 2, 2, 4), (2, 2, 2, 2), (4, 2, 2, 1)]
    H = oracle.chain(np.eye(8), [hadamard_values(p) for p in pats], pats)
    np.testing.assert_array_equal(H, H8)


def test_golden_hand_examples():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 4
    for case in cases:
        Y = oracle.matmul(np.array(case["X"], dtype=float), np.array(case["values"], dtype=float),
                          tuple(case["pattern"]))
        np.testing.assert_array_equal(Y, np.array(case["Y"], dtype=float), err_msg=case["name"])


def test_empty_batch():
    assert oracle.matmul(np.zeros((0, 8)), np.ones(16), (2, 2, 2, 2)).shape == (0, 8)


def test_threads_do_not_change_results():
    X, V = rand_case((2, 4, 4, 2), n=64, seed=5)
    oracle.set_threads(1)
    Y1 = oracle.matmul(X, V, (2, 4, 4, 2))
    oracle.set_threads(4)
    Y4 = oracle.matmul(X, V, (2, 4, 4, 2))
    oracle.set_threads(0)
    np.testing.assert_array_equal(Y1, Y4)


def test_max_rel_err():
    assert oracle.max_rel_err(np.array([1.0, 2.0]), np.array([1.0, 4.0])) == 0.5
