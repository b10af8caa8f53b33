"""Plant plausible mistakes in a copy of the oracle (on the CPU, in a temporary
directory) and check that the pins of test_oracle.py catch every one of them:
a dropped term, a wrong sign, swapped or transposed indices.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from tests.test_oracle import TINY, kron_dense, rand_case

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ks_ref.c")

MUTANTS = {
    "dropped_first_term": ("for (int64_t j = 0; j < c; ++j)\n                        acc +=",
                           "for (int64_t j = 1; j < c; ++j)\n                        acc +="),
    "wrong_sign": ("acc += values", "acc -= values"),
    "output_k_l_swapped": ("y[i * b * d + k * d + l] = acc", "y[i * b * d + l * b + k] = acc"),
    "input_j_l_swapped": ("x[i * c * d + j * d + l]", "x[i * c * d + l * c + j]"),
    "values_transposed": ("values[((i * d + l) * b + k) * c + j] *",
                          "values[((i * d + l) * c + j) * b + k] *"),
    "values_l_k_order": ("values[((i * d + l) * b + k) * c + j] *",
                         "values[((i * b + k) * d + l) * c + j] *"),
    "block_offset_dropped": ("x[i * c * d + j * d + l]", "x[j * d + l]"),
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
    lib.ks_ref_matmul.argtypes = [dp, dp] + [ctypes.c_int64] * 5 + [dp]
    return lib


def mutant_matmul(lib, X, V, p):
    a, b, c, d = p
    X = np.ascontiguousarray(X, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64).reshape(-1)
    Y = np.zeros((X.shape[0], a * b * d))
    dp = ctypes.POINTER(ctypes.c_double)
    lib.ks_ref_matmul(X.ctypes.data_as(dp), V.ctypes.data_as(dp), a, b, c, d, X.shape[0],
                      Y.ctypes.data_as(dp))
    return Y


def pins_pass(lib):
    for p in TINY:
        X, V = rand_case(p, seed=sum(p))
        if not np.allclose(mutant_matmul(lib, X, V, p), X @ kron_dense(V, p).T, rtol=1e-12, atol=1e-12):
            return False
    return True


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    assert not pins_pass(build_mutant(tmp_path, name))
