"""Pins for the oracle's hierarchical butterfly factorization: exact
recovery of products of random butterfly factors (the product computed by
the oracle's chain, itself pinned to numpy's Kronecker product), the
Sylvester-Hadamard closed form, the rank-one block structure of a
two-factor product, and planted mistakes that must break a pin."""
import math
import os
import types

import numpy as np
import pytest

import oracle
from oracle import factorize
from kronecker_sparse_matrix_b200.inputs import butterfly_patterns

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "factorize.py")


def dense_of(factors, L):
    """K of Y = X K^T for the chain F_1 first: K = chain(I)^T."""
    return oracle.chain(np.eye(2 ** L), factors, butterfly_patterns(L)).T


def random_butterfly(L, seed):
    r = np.random.default_rng(seed)
    return [r.standard_normal(int(np.prod(p))) for p in butterfly_patterns(L)]


def recovery_error(mod, L, seed):
    K = dense_of(random_butterfly(L, seed), L)
    rec = mod.hierarchical_butterfly(K)
    return np.max(np.abs(dense_of(rec, L) - K)) / np.max(np.abs(K))


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 6, 7])
def test_exact_recovery_of_butterfly_products(L):
    assert recovery_error(factorize, L, seed=L) < 1e-10


def test_sylvester_hadamard():
    L = 6
    r = np.arange(2 ** L)
    H = np.array([[(-1.0) ** bin(x & y).count("1") for y in r] for x in r])
    rec = factorize.hierarchical_butterfly(H)
    np.testing.assert_allclose(dense_of(rec, L), H, atol=1e-10)
    # every factor of H is made of scaled 2 x 2 Hadamard blocks up to signs: |entries| equal per factor
    for v in rec:
        a = np.abs(v)
        assert np.allclose(a, a[0])


def test_range_patterns_chain():
    L = 12
    for p in range(1, L + 1):
        for q in range(p, L + 1):
            a, b, c, d = factorize.butterfly_range_pattern(p, q, L)
            assert a * b * d == 2 ** L and a * c * d == 2 ** L
            if p == q:
                assert (a, b, c, d) == butterfly_patterns(L)[p - 1]


def test_two_factor_blocks_are_rank_one_products():
    # a product of two chainable KS factors is fitted exactly, and refitting
    # the fit changes nothing
    p1, p2 = (2, 3, 2, 4), (6, 2, 2, 2)  # a2 = a1*b1, d1 = c2*d2
    r = np.random.default_rng(3)
    V1 = r.standard_normal(int(np.prod(p1)))
    V2 = r.standard_normal(int(np.prod(p2)))
    K = oracle.densify(V2, p2) @ oracle.densify(V1, p1)  # K2 K1
    a1, b1, c1, d1 = p1
    a2, b2, c2, d2 = p2
    prod = (a1, b1 * b2, c1 * c2, d2)
    # the product's values: read K at the product pattern's support
    Pv = np.zeros(int(np.prod(prod)))
    for e in range(Pv.size):
        unit = np.zeros(Pv.size)
        unit[e] = 1.0
        Pv[e] = np.sum(oracle.densify(unit, prod) * K)
    W1, W2 = factorize.two_factor(Pv, p1, p2)
    np.testing.assert_allclose(oracle.densify(W2, p2) @ oracle.densify(W1, p1), K, atol=1e-12)
    X1, X2 = factorize.two_factor(Pv, p1, p2)
    np.testing.assert_array_equal(W1, X1)


def test_best_rank_one_is_a_singular_pair():
    B = np.random.default_rng(5).standard_normal((7, 5))
    s, u, v = factorize.rank_one(B)
    np.testing.assert_allclose(B @ v, s * u, atol=1e-12)
    np.testing.assert_allclose(B.T @ u, s * v, atol=1e-12)
    # largest: no unit vector w gives |B w| > s (checked on many random w)
    W = np.random.default_rng(6).standard_normal((5, 2000))
    W /= np.linalg.norm(W, axis=0)
    assert np.max(np.linalg.norm(B @ W, axis=0)) <= s * (1 + 1e-12)
    assert math.isclose(np.linalg.norm(u), 1.0) and v[np.argmax(np.abs(v))] > 0


MUTANTS = {
    "j_digits_swapped": ("P[i1, l2, k1 * b2:(k1 + 1) * b2, j2::c2]", "P[i1, l2, k1 * b2:(k1 + 1) * b2, j2 * c1:(j2 + 1) * c1]"),
    "v1_l_order": ("V1[i1, j2 * d2 + l2, k1, :]", "V1[i1, l2 * c2 + j2, k1, :]"),
    "no_sqrt_split": ("V1[i1, j2 * d2 + l2, k1, :] = np.sqrt(s) * v", "V1[i1, j2 * d2 + l2, k1, :] = v"),
    "v2_block_index": ("V2[i1 * b1 + k1, l2, :, j2]", "V2[k1 * a1 + i1, l2, :, j2]"),
    "split_point": ("r = (p + q - 1) // 2", "r = (p + q + 1) // 2"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1
    mod = types.ModuleType("mutant")
    try:
        exec(compile(src.replace(old, new), "mutant", "exec"), mod.__dict__)
        bad = any(recovery_error(mod, L, seed=L) > 1e-6 for L in (2, 3, 4, 5))
    except Exception:
        bad = True
    assert bad
