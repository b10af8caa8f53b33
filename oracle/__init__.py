"""Plain CPU oracle for Kronecker-sparse (KS) matrix multiplication.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``kronecker_sparse_matrix_b200``) never imports it, and it imports nothing
from the product path.

The arithmetic lives in ``ks_ref.c`` (double precision, the definition written
out as loops); this module only marshals numpy arrays to it.  Its source is the
taxoreview.com page on Kronecker-sparse matrix multiplication (first abstract:
supports are Kronecker products of identity and all-ones blocks; butterfly and
Monarch matrices are products of such factors), read with the textbook
Kronecker index order:

    K[i*b*d + k*d + l, i*c*d + j*d + l] = values[i, l, k, j],
    Y[n, i*b*d + k*d + l] = sum_j values[i, l, k, j] * X[n, i*c*d + j*d + l].

Every function here is pinned by ``tests/test_oracle.py`` against things the
oracle does not compute itself (numpy's Kronecker product, numpy/torch matrix
products, the Sylvester-Hadamard closed form, hand-worked fixtures).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ks_ref.c")
_LIB_PATH = os.path.join(_HERE, "libks_ref.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ``ks_ref.c`` into ``libks_ref.so`` beside it (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.ks_ref_matmul.argtypes = [_dp, _dp, _i64, _i64, _i64, _i64, _i64, _dp]
            lib.ks_ref_matmul.restype = None
            lib.ks_ref_densify.argtypes = [_dp, _i64, _i64, _i64, _i64, _dp]
            lib.ks_ref_densify.restype = None
            lib.ks_ref_dense_matmul.argtypes = [_dp, _dp, _i64, _i64, _i64, _dp]
            lib.ks_ref_dense_matmul.restype = None
            lib.ks_ref_chain.argtypes = [_dp, ctypes.POINTER(_dp),
                                         ctypes.POINTER(_i64), ctypes.c_int, _i64, _dp]
            lib.ks_ref_chain.restype = ctypes.c_int
            lib.ks_ref_dx.argtypes = [_dp, _dp, _i64, _i64, _i64, _i64, _i64, _dp]
            lib.ks_ref_dx.restype = None
            lib.ks_ref_dv.argtypes = [_dp, _dp, _i64, _i64, _i64, _i64, _i64, _dp]
            lib.ks_ref_dv.restype = None
            lib.ks_ref_set_threads.argtypes = [ctypes.c_int]
            lib.ks_ref_set_threads.restype = None
            lib.ks_ref_get_threads.argtypes = []
            lib.ks_ref_get_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Exact conversion to a C-contiguous float64 array (torch tensors too)."""
    if hasattr(a, "detach"):  # torch tensor: fp32 / bf16 / fp64 values are exact in fp64
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def set_threads(n: int) -> None:
    """Threads the oracle's outer loop over batch rows may use (<=0: default)."""
    _load().ks_ref_set_threads(int(n))


def threads() -> int:
    return int(_load().ks_ref_get_threads())


def _check_pattern(pattern):
    a, b, c, d = (int(v) for v in pattern)
    if min(a, b, c, d) <= 0:
        raise ValueError(f"pattern entries must be positive, got {pattern}")
    return a, b, c, d


def matmul(X, values, pattern) -> np.ndarray:
    """Y = X K^T for one KS factor; X is (N, a*c*d), values is [a][d][b][c]."""
    a, b, c, d = _check_pattern(pattern)
    X = _f64(X)
    V = _f64(values).reshape(-1)
    if V.size != a * b * c * d:
        raise ValueError("values must hold a*b*c*d entries")
    X = X.reshape(-1, a * c * d) if X.size else X.reshape(0, a * c * d)
    N = X.shape[0]
    Y = np.zeros((N, a * b * d), dtype=np.float64)
    if N:
        _load().ks_ref_matmul(_ptr(X), _ptr(V), a, b, c, d, N, _ptr(Y))
    return Y


def dx(dY, values, pattern) -> np.ndarray:
    """Input gradient of Y = X K^T: dX = dY K, (N, a*c*d) from dY (N, a*b*d)."""
    a, b, c, d = _check_pattern(pattern)
    G = _f64(dY)
    V = _f64(values).reshape(-1)
    if V.size != a * b * c * d:
        raise ValueError("values must hold a*b*c*d entries")
    G = G.reshape(-1, a * b * d) if G.size else G.reshape(0, a * b * d)
    N = G.shape[0]
    H = np.zeros((N, a * c * d), dtype=np.float64)
    if N:
        _load().ks_ref_dx(_ptr(G), _ptr(V), a, b, c, d, N, _ptr(H))
    return H


def dv(dY, X, pattern) -> np.ndarray:
    """Values gradient of Y = X K^T: dV[i][l][k][j] = sum_n dY[n,(i,k,l)] X[n,(i,j,l)],
    returned flat in the values layout [a][d][b][c]."""
    a, b, c, d = _check_pattern(pattern)
    G = _f64(dY)
    X = _f64(X)
    G = G.reshape(-1, a * b * d) if G.size else G.reshape(0, a * b * d)
    X = X.reshape(-1, a * c * d) if X.size else X.reshape(0, a * c * d)
    if G.shape[0] != X.shape[0]:
        raise ValueError("dY and X need the same number of rows")
    dV = np.zeros(a * b * c * d, dtype=np.float64)
    _load().ks_ref_dv(_ptr(G), _ptr(X), a, b, c, d, G.shape[0], _ptr(dV))
    return dV


def bias_grad(dY) -> np.ndarray:
    """Bias gradient of y = x K^T + bias: db[col] = sum_n dY[n][col] (the bias
    is added to every row), summed in fp64; zeros for an empty batch."""
    G = _f64(dY)
    if G.ndim != 2:
        raise ValueError("dY must be batch x width")
    return G.sum(axis=0) if G.shape[0] else np.zeros(G.shape[1], dtype=np.float64)


def densify(values, pattern) -> np.ndarray:
    """The dense (a*b*d, a*c*d) matrix K of one factor."""
    a, b, c, d = _check_pattern(pattern)
    V = _f64(values).reshape(-1)
    if V.size != a * b * c * d:
        raise ValueError("values must hold a*b*c*d entries")
    K = np.zeros((a * b * d, a * c * d), dtype=np.float64)
    _load().ks_ref_densify(_ptr(V), a, b, c, d, _ptr(K))
    return K


def dense_matmul(X, K) -> np.ndarray:
    """Y = X K^T for a dense K, by the naive triple loop."""
    X = _f64(X)
    K = _f64(K)
    rows, cols = K.shape
    X = X.reshape(-1, cols)
    Y = np.zeros((X.shape[0], rows), dtype=np.float64)
    if X.shape[0]:
        _load().ks_ref_dense_matmul(_ptr(X), _ptr(K), X.shape[0], rows, cols, _ptr(Y))
    return Y


def chain(X, factors, patterns) -> np.ndarray:
    """Apply the factors in order (factor 0 first): Y = X (K_{n-1}...K_0)^T."""
    pats = [_check_pattern(p) for p in patterns]
    if len(pats) != len(factors) or not pats:
        raise ValueError("need one pattern per factor and at least one factor")
    Vs = [_f64(v).reshape(-1) for v in factors]
    for V, (a, b, c, d) in zip(Vs, pats):
        if V.size != a * b * c * d:
            raise ValueError("a factor's values must hold a*b*c*d entries")
    a0, b0, c0, d0 = pats[0]
    X = _f64(X).reshape(-1, a0 * c0 * d0)
    a1, b1, c1, d1 = pats[-1]
    Y = np.zeros((X.shape[0], a1 * b1 * d1), dtype=np.float64)
    ptrs = (_dp * len(Vs))(*[_ptr(V) for V in Vs])
    flat = (_i64 * (4 * len(pats)))(*[v for p in pats for v in p])
    if X.shape[0]:
        rc = _load().ks_ref_chain(_ptr(X), ptrs, flat, len(pats), X.shape[0], _ptr(Y))
        if rc != 0:
            raise ValueError("chain widths do not match (a*b*d of factor t must equal "
                             "a*c*d of factor t+1)")
    return Y


ACTIVATIONS = ("none", "relu", "gelu_tanh", "gelu_erf")


def activation(Z, act: str) -> np.ndarray:
    """The pointwise activations of the MLP shapes, on fp64 values, from their
    definitions: relu(z) = max(z, 0); gelu_erf(z) = z * Phi(z) with
    Phi(z) = (1 + erf(z / sqrt 2)) / 2; gelu_tanh(z) = z (1 + tanh(sqrt(2/pi)
    (z + 0.044715 z^3))) / 2, the usual tanh form of the same function."""
    Z = _f64(Z)
    if act == "none":
        return Z.copy()
    if act == "relu":
        return np.maximum(Z, 0.0)
    if act == "gelu_erf":
        erf = np.vectorize(math.erf, otypes=[np.float64])
        return 0.5 * Z * (1.0 + erf(Z / math.sqrt(2.0)))
    if act == "gelu_tanh":
        return 0.5 * Z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (Z + 0.044715 * Z ** 3)))
    raise ValueError(f"unknown activation {act!r}")


def matmul_epilogue(X, values, pattern, bias=None, act: str = "none") -> np.ndarray:
    """act(X K^T + bias): the product, plus bias[col] on every row (bias has
    a*b*d entries, or None), then the activation, all in fp64."""
    Y = matmul(X, values, pattern)
    if bias is not None:
        B = _f64(bias).reshape(-1)
        if B.size != Y.shape[1]:
            raise ValueError("bias must hold a*b*d entries")
        Y = Y + B[None, :]
    return activation(Y, act)


def max_rel_err(Y, Y_ref) -> float:
    """max|Y - Y_ref| / max|Y_ref| (0 when both are empty)."""
    Y = _f64(Y)
    Y_ref = _f64(Y_ref)
    if Y_ref.size == 0:
        return 0.0
    den = float(np.max(np.abs(Y_ref)))
    num = float(np.max(np.abs(Y - Y_ref)))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den
