"""CPU models of the fused epilogue's GELU arithmetic (no GPU).

The kernels evaluate GELU in its tanh form through algebraic rewrites of the
definition z (1 + tanh(u)) / 2, u = sqrt(2/pi) (z + 0.044715 z^3):

- fp32 kernels (ks_epilogue.cuh): z / (1 + 2^s), s = z (A + B z^2) with
  A = -2 log2(e) sqrt(2/pi), B = 0.044715 A (the logistic form, through the
  PTX ex2.approx and rcp.approx instructions);
- tensor-core epilogue (ks_tc.cu): h + h tanh(z (c0 + c1 z^2)), h = z / 2,
  with the literals c0, c1 written in the kernel.

The constants are read from the sources, the steps are replayed in float32
(ex2 and the reciprocal as exact float32 operations, overflow to inf
included) and compared with the oracle's fp64 definition over a range that
takes 2^s past overflow, so a wrong constant, a lost factor or a sign slip
fails here before any kernel runs.
"""
import os
import re

import numpy as np

import oracle

CSRC = os.path.join(os.path.dirname(__file__), "..", "kronecker_sparse_matrix_b200", "csrc")
F = np.float32


def _src(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def _floats(expr):
    return [F(float(x)) for x in re.findall(r"([0-9]*\.[0-9]+(?:e-?[0-9]+)?)f", expr)]


def _product(expr):
    """Value of a constexpr product of float literals, one rounding per multiply."""
    sign = F(-1.0) if expr.strip().startswith("-") else F(1.0)
    v = sign
    for x in _floats(expr):
        v = F(v * x)
    return v


def _fp32_gelu_constants():
    s = _src("ks_epilogue.cuh")
    a = re.search(r"constexpr float kGeluA = ([^;]+);", s).group(1)
    b = re.search(r"constexpr float kGeluB = ([^;]+);", s).group(1)
    A = _product(a)
    assert b.replace(" ", "").endswith("*kGeluA")
    B = F(_floats(b)[0] * A)
    return A, B


def _tc_gelu_constants():
    s = _src("ks_tc.cu")
    m = re.search(r"__ffma2_rn\(z2, make_float2\(([0-9.]+)f, \1f\),\s*make_float2\(([0-9.]+)f, \2f\)\)", s)
    assert m, "packed GELU of the tensor-core epilogue not found"
    return F(float(m.group(2))), F(float(m.group(1)))  # c0, c1


def _z_grid():
    z = np.concatenate([np.linspace(-40, 40, 8001), [-1e4, -200, -90, -12, -10.5, -10, 0.0, 1e-30, 10, 90, 1e4]])
    return z.astype(np.float32)


def test_fp32_logistic_form_constants_match_the_definition():
    A, B = _fp32_gelu_constants()
    assert abs(float(A) - (-2 * np.log2(np.e) * np.sqrt(2 / np.pi))) < 1e-6
    assert abs(float(B) - 0.044715 * float(A)) < 1e-7


def test_fp32_logistic_form_matches_the_oracle_including_overflow():
    A, B = _fp32_gelu_constants()
    z = _z_grid()
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        s = F(1) * z * (F(1) * z * z * B + A)           # z * fma(z*z, B, A), float32 steps
        s = s.astype(np.float32)
        den = (np.exp2(s.astype(np.float32)) + F(1)).astype(np.float32)
        y = (z * (F(1) / den)).astype(np.float32)
    ref = oracle.activation(z.astype(np.float64), "gelu_tanh")
    assert np.all(np.isfinite(y))
    err = np.abs(y.astype(np.float64) - ref)
    # a few float32 ulps of the output, or of 1 near zero
    assert np.all(err <= 4e-6 * np.abs(ref) + 1e-7), float(np.max(err / (np.abs(ref) + 1e-30)))
    # the two overflow sides: very negative z -> 2^s = inf -> -0, very positive -> z
    assert y[z == F(-1e4)][0] == 0.0 and y[z == F(1e4)][0] == F(1e4)


def test_tc_packed_form_constants_and_values():
    c0, c1 = _tc_gelu_constants()
    assert abs(float(c0) - np.sqrt(2 / np.pi)) < 1e-7
    assert abs(float(c1) - 0.044715 * np.sqrt(2 / np.pi)) < 1e-8
    z = _z_grid()
    with np.errstate(over="ignore", invalid="ignore"):
        u = (z * ((z * z).astype(np.float32) * c1 + c0)).astype(np.float32)
        h = (z * F(0.5)).astype(np.float32)
        y = (h * np.tanh(u).astype(np.float32) + h).astype(np.float32)
    ref = oracle.activation(z.astype(np.float64), "gelu_tanh")
    assert np.all(np.isfinite(y))
    # exact tanh here: only float32 rounding separates the two (the kernel's
    # tanh.approx adds about 2^-11 relative, inside the bf16 / TF32 tolerances)
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(err <= 4e-6 * np.abs(z) + 1e-7), float(np.max(err))
