"""Hierarchical butterfly factorization on the GPU (ks_butterfly_factorize)
against the oracle's factorization of the same matrix.  The targets are
products of random butterfly factors built by the oracle, so every block of
every split is exactly rank one and the fit is unique (the sqrt(s) split and
the sign rule fix the scale and sign): factors compare element by element.
Tolerance 1e-4 relative to the factor's largest entry: fp32 rounding passes
through up to four levels of splits (log2 of 12) and a power iteration.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import factorize
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def target(L, seed):
    r = np.random.default_rng(seed)
    pats = inputs.butterfly_patterns(L)
    facs = [r.standard_normal(int(np.prod(p))) * np.sqrt(0.5) for p in pats]
    return np.ascontiguousarray(oracle.chain(np.eye(2 ** L), facs, pats).T)  # K of Y = X K^T


@pytest.mark.parametrize("L", [2, 3, 5, 8, 10, 12])
def test_factors_match_oracle(L):
    K = target(L, seed=L)
    ref = factorize.hierarchical_butterfly(K)
    got, pats = ks.butterfly_factorize(torch.tensor(K, dtype=torch.float32, device=DEV))
    ks.sync_status()
    assert pats == inputs.butterfly_patterns(L)
    for g, r in zip(got, ref):
        assert oracle.max_rel_err(g.cpu(), r) <= 1e-4
    if L <= 10:  # the product of the fitted factors is the target
        prod = oracle.chain(np.eye(2 ** L), [g.cpu() for g in got], pats).T
        assert oracle.max_rel_err(prod, K) <= 1e-5


def test_hadamard():
    L = 8
    r = np.arange(2 ** L)
    H = np.array([[(-1.0) ** bin(x & y).count("1") for y in r] for x in r])
    got, pats = ks.butterfly_factorize(torch.tensor(H, dtype=torch.float32, device=DEV))
    ks.sync_status()
    prod = oracle.chain(np.eye(2 ** L), [g.cpu() for g in got], pats).T
    assert np.max(np.abs(prod - H)) <= 1e-5


def test_factorized_chain_applies_the_matrix():
    # the factors feed the fused butterfly chain: X A^T through 12 factors
    L = 12
    K = target(L, seed=99)
    got, pats = ks.butterfly_factorize(torch.tensor(K, dtype=torch.float32, device=DEV))
    X = torch.randn(64, 4096, generator=torch.Generator().manual_seed(1))
    Y = ks.chain(X.to(DEV), got, pats)
    ks.sync_status()
    assert oracle.max_rel_err(Y.cpu(), X.double().numpy() @ K.T) <= 1e-4


def test_factorize_argument_errors():
    a = torch.zeros(6, 6, device=DEV)
    with pytest.raises(ValueError):
        ks.butterfly_factorize(a)
    with pytest.raises(ks.KsError) as e:
        ks.butterfly_factorize(torch.zeros(8, 8, dtype=torch.bfloat16, device=DEV))
    assert e.value.status == 3
