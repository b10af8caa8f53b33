"""Chains of KS factors on the GPU against the oracle's chain (which is pinned
to the densified product and to the Sylvester-Hadamard closed form)."""
import numpy as np
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_hadamard_chain_is_exact():
    m = 8
    pats = inputs.butterfly_patterns(m)
    h2 = torch.tensor([[1.0, 1.0], [1.0, -1.0]])
    facs = [h2.expand(p[0], p[3], 2, 2).contiguous().to(DEV) for p in pats]
    Y = ks.chain(torch.eye(2 ** m, device=DEV), facs, pats).cpu().numpy()
    r = np.arange(2 ** m)
    closed = np.array([[(-1.0) ** bin(x & y).count("1") for y in r] for x in r])
    np.testing.assert_array_equal(Y, closed)


@pytest.mark.parametrize("patterns", [
    [(1, 2, 2, 4), (2, 2, 2, 2), (4, 2, 2, 1)],
    [(4, 64, 64, 1), (1, 64, 64, 4)],                    # Monarch-like, 256 wide
    [(2, 96, 48, 1), (1, 48, 192, 1), (3, 16, 16, 1)],   # rectangular 96 -> 192 -> 48 -> 48
    [(1, 192, 48, 8), (8, 48, 192, 1)],                  # 384 -> 1536 -> 384
])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_small_chains(patterns, dtype):
    c = inputs.chain_inputs(patterns, 45, seed=4, dtype=dtype)
    Y = ks.chain(c.X.to(DEV), [f.to(DEV) for f in c.factors], patterns)
    ks.sync_status()
    ref = oracle.chain(c.X, c.factors, patterns)
    tol = 1e-5 if dtype == torch.float32 else 3e-2  # bf16: one rounding per factor
    assert oracle.max_rel_err(Y.cpu(), ref) <= tol


def test_butterfly_chain_full_size_sampled_rows():
    c = inputs.butterfly(device=DEV)
    Y = ks.chain(c.X, c.factors, c.patterns)
    ks.sync_status()
    rows = [0, 1, 17, 1000, 2048, 4095]
    ref = oracle.chain(c.X[rows].cpu(), [f.cpu() for f in c.factors], c.patterns)
    assert oracle.max_rel_err(Y[rows].cpu(), ref) <= 1e-5


def test_chain_of_one_equals_matmul():
    f = inputs.factor_inputs((2, 64, 64, 2), 30)
    X, V = f.X.to(DEV), f.values.to(DEV)
    assert torch.equal(ks.chain(X, [V], [(2, 64, 64, 2)]), ks.matmul(X, V, (2, 64, 64, 2)))
