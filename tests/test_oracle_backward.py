"""Pins for the oracle's two gradients of Y = X K^T (the page's KSLinear layer
is trained through them): dX = dY K and dV[i][l][k][j] = sum_n dY[n,(i,k,l)]
X[n,(i,j,l)].  Each check compares them with something they do not compute
themselves: numpy products with K built from numpy's Kronecker product, the
adjoint identity <X K^T, G> = <X, G K>, the linearity of the loss in the values,
and a closed form.  Planted mistakes in a copy of the C source must fail a pin.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from tests.test_oracle import TINY, kron_dense, rand_case

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ks_ref.c")


def grad_case(pattern, n=4, seed=0):
    a, b, c, d = pattern
    X, V = rand_case(pattern, n=n, seed=seed)
    G = np.random.default_rng(seed + 1000).standard_normal((n, a * b * d))
    return X, V, G


def support_entries(D, pattern):
    """The entries of a dense (a*b*d, a*c*d) matrix at K's support, in the
    values layout, located through numpy's Kronecker product of the support."""
    a, b, c, d = pattern
    out = np.zeros((a, d, b, c))
    for i in range(a):
        for l in range(d):
            for k in range(b):
                for j in range(c):
                    unit = np.zeros((a, d, b, c))
                    unit[i, l, k, j] = 1.0
                    out[i, l, k, j] = np.sum(kron_dense(unit, pattern) * D)
    return out.reshape(-1)


@pytest.mark.parametrize("pattern", TINY)
def test_dx_is_dense_gradient(pattern):
    X, V, G = grad_case(pattern, seed=sum(pattern))
    K = kron_dense(V, pattern)
    np.testing.assert_allclose(oracle.dx(G, V, pattern), G @ K, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pattern", [p for p in TINY if np.prod(p) <= 24])
def test_dv_is_dense_gradient_on_the_support(pattern):
    X, V, G = grad_case(pattern, n=6, seed=sum(pattern) + 1)
    np.testing.assert_allclose(oracle.dv(G, X, pattern), support_entries(G.T @ X, pattern),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pattern", [(2, 3, 4, 2), (1, 5, 3, 1), (3, 2, 2, 4), (2, 4, 4, 2)])
def test_adjoint_identity(pattern):
    X, V, G = grad_case(pattern, n=7, seed=3)
    lhs = np.sum(oracle.matmul(X, V, pattern) * G)
    rhs = np.sum(X * oracle.dx(G, V, pattern))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


@pytest.mark.parametrize("pattern", [(2, 3, 4, 2), (1, 5, 3, 1), (3, 2, 2, 4), (2, 4, 4, 2)])
def test_dv_is_the_derivative_of_a_linear_loss(pattern):
    # L(V) = <X K(V)^T, G> is linear in V, so <dV, E> = L(E) for any direction E.
    X, V, G = grad_case(pattern, n=9, seed=5)
    E = np.random.default_rng(11).standard_normal(V.size)
    lhs = np.sum(oracle.dv(G, X, pattern) * E)
    rhs = np.sum(oracle.matmul(X, E, pattern) * G)
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_diagonal_closed_forms():
    # b = c = 1: K is diagonal with entries values[i][l] at (i, l), so
    # dX = dY * v and dV = sum_n dY * X columnwise.
    a, d = 3, 4
    r = np.random.default_rng(2)
    v = r.standard_normal(a * d)
    G = r.standard_normal((5, a * d))
    X = r.standard_normal((5, a * d))
    np.testing.assert_allclose(oracle.dx(G, v, (a, 1, 1, d)), G * v, rtol=1e-14)
    np.testing.assert_allclose(oracle.dv(G, X, (a, 1, 1, d)), np.sum(G * X, axis=0), rtol=1e-13)


def test_empty_batch_gives_zero_gradient():
    p = (2, 3, 4, 2)
    np.testing.assert_array_equal(oracle.dv(np.zeros((0, 12)), np.zeros((0, 16)), p), np.zeros(48))
    assert oracle.dx(np.zeros((0, 12)), np.ones(48), p).shape == (0, 16)


MUTANTS = {
    "dx_dropped_last_term": ("for (int64_t k = 0; k < b; ++k)\n                        acc += g[",
                             "for (int64_t k = 0; k + 1 < b; ++k)\n                        acc += g["),
    "dx_values_not_transposed": ("values[(i * d + l) * b * c + k * c + j]",
                                 "values[(i * d + l) * b * c + j * b + k]"),
    "dx_output_j_l_swapped": ("h[i * c * d + j * d + l] = acc", "h[i * c * d + l * c + j] = acc"),
    "dv_wrong_operand_row": ("X[n * in_f + i * c * d + j * d + l]", "X[n * in_f + i * c * d + k * d + l]"),
    "dv_layout_k_j_swapped": ("dV[((i * d + l) * b + k) * c + j] = acc", "dV[((i * d + l) * c + j) * b + k] = acc"),
    "dv_first_row_dropped": ("for (int64_t n = 0; n < N; ++n)\n                    acc += dY",
                             "for (int64_t n = 1; n < N; ++n)\n                    acc += dY"),
}


def build_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(path)], check=True)
    lib = ctypes.CDLL(str(so))
    dp = ctypes.POINTER(ctypes.c_double)
    for f in (lib.ks_ref_dx, lib.ks_ref_dv):
        f.argtypes = [dp, dp] + [ctypes.c_int64] * 5 + [dp]
    return lib


def _call(f, A, B, p, out_size):
    dp = ctypes.POINTER(ctypes.c_double)
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    out = np.zeros(out_size)
    f(A.ctypes.data_as(dp), B.ctypes.data_as(dp), *p, A.shape[0], out.ctypes.data_as(dp))
    return out


def pins_pass(lib):
    for p in [q for q in TINY if np.prod(q) <= 24]:
        a, b, c, d = p
        X, V, G = grad_case(p, n=6, seed=sum(p) + 1)
        dx = _call(lib.ks_ref_dx, G, V, p, G.shape[0] * a * c * d).reshape(G.shape[0], -1)
        if not np.allclose(dx, G @ kron_dense(V, p), rtol=1e-12, atol=1e-12):
            return False
        dv = _call(lib.ks_ref_dv, G, X, p, a * b * c * d)
        if not np.allclose(dv, support_entries(G.T @ X, p), rtol=1e-12, atol=1e-12):
            return False
    return True


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_pins_catch_planted_mistake(tmp_path, name):
    assert not pins_pass(build_mutant(tmp_path, name))


def test_bias_grad_closed_forms_and_the_epilogue_derivative():
    # ones: every column sums to the batch; row n = n + 1: batch (batch + 1) / 2
    np.testing.assert_array_equal(oracle.bias_grad(np.ones((7, 3))), [7.0, 7.0, 7.0])
    rows = np.arange(1, 11, dtype=float)[:, None] * np.ones((1, 4))
    np.testing.assert_array_equal(oracle.bias_grad(rows), [55.0] * 4)
    np.testing.assert_array_equal(oracle.bias_grad(np.zeros((0, 5))), np.zeros(5))
    # db is the derivative of L(b) = <act-free epilogue(X, V, b), G> in b: L is
    # linear in b, so L(b + t e_col) - L(b) = t db[col] exactly (t a power of two)
    p = (2, 3, 4, 2)
    rng = np.random.default_rng(3)
    X = rng.integers(-3, 4, size=(5, 2 * 4 * 2)).astype(float)
    V = rng.integers(-3, 4, size=2 * 3 * 4 * 2).astype(float)
    G = rng.integers(-3, 4, size=(5, 2 * 3 * 2)).astype(float)
    b = rng.integers(-3, 4, size=2 * 3 * 2).astype(float)
    L = lambda bb: float(np.sum(oracle.matmul_epilogue(X, V, p, bb, "none") * G))
    db = oracle.bias_grad(G)
    for col in range(b.size):
        e = np.zeros_like(b)
        e[col] = 0.5
        assert L(b + e) - L(b) == 0.5 * db[col]
