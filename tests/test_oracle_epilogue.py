"""Pins for the oracle's epilogue (bias and activation after a KS product,
the fused epilogue of the MLP shapes): values of the activations against
scipy's normal distribution and closed forms, and the epilogue against the
plain product plus bias."""
import math

import numpy as np
import pytest
from scipy import special, stats

import oracle
from tests.test_oracle import rand_case


def test_relu_closed_form():
    z = np.array([-2.5, -0.0, 0.0, 1e-30, 3.25])
    np.testing.assert_array_equal(oracle.activation(z, "relu"), [0.0, 0.0, 0.0, 1e-30, 3.25])


def test_gelu_erf_is_z_times_normal_cdf():
    z = np.linspace(-6, 6, 97)
    np.testing.assert_allclose(oracle.activation(z, "gelu_erf"), z * stats.norm.cdf(z), rtol=1e-13, atol=1e-15)


def test_gelu_tanh_form():
    z = np.linspace(-6, 6, 97)
    ref = 0.5 * z * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (z + 0.044715 * z ** 3)))
    np.testing.assert_allclose(oracle.activation(z, "gelu_tanh"), ref, rtol=1e-14, atol=1e-15)
    # the tanh form approximates z Phi(z) to within 1e-3 everywhere
    assert np.max(np.abs(oracle.activation(z, "gelu_tanh") - z * stats.norm.cdf(z))) < 1e-3


def test_gelu_special_values():
    assert oracle.activation(np.array([0.0]), "gelu_erf")[0] == 0.0
    # gelu(1) = Phi(1) = (1 + erf(1/sqrt 2)) / 2
    assert abs(oracle.activation(np.array([1.0]), "gelu_erf")[0] - 0.5 * (1 + special.erf(1 / math.sqrt(2)))) < 1e-15
    # odd part: gelu(z) - gelu(-z) = z
    z = np.linspace(-3, 3, 13)
    np.testing.assert_allclose(oracle.activation(z, "gelu_erf") - oracle.activation(-z, "gelu_erf"), z, atol=1e-14)


@pytest.mark.parametrize("act", oracle.ACTIVATIONS)
def test_epilogue_is_product_plus_bias_then_activation(act):
    p = (2, 3, 4, 2)
    X, V = rand_case(p, n=6, seed=4)
    bias = np.random.default_rng(9).standard_normal(2 * 3 * 2)
    Z = oracle.matmul(X, V, p) + bias[None, :]
    np.testing.assert_allclose(oracle.matmul_epilogue(X, V, p, bias, act), oracle.activation(Z, act), rtol=0, atol=0)
    np.testing.assert_allclose(oracle.matmul_epilogue(X, V, p, None, "none"), oracle.matmul(X, V, p), rtol=0, atol=0)


def test_epilogue_matches_hand_worked_examples():
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "epilogue_examples.json")
    for case in json.load(open(path))["cases"]:
        p = tuple(case["pattern"])
        got = oracle.matmul_epilogue(np.array(case["X"], dtype=float), np.array(case["values"], dtype=float), p,
                                     np.array(case["bias"], dtype=float), case["act"])
        np.testing.assert_array_equal(got, np.array(case["Y"], dtype=float), err_msg=case["name"])
