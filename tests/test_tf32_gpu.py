"""KS_TF32 on the tcgen05 tensor cores (kind::tf32): fp32 buffers, TF32
operands, fp32 accumulation, against the oracle at the TF32 tolerance
max|Y - Y_ref| / max|Y_ref| <= 5e-3, element by element on the same seeded
inputs, through the C ABI.

The tolerance covers TF32's 10 explicit mantissa bits: each operand is read
with a relative error below 2^-10, so every product carries at most about
2 * 2^-10 = 2e-3 of relative error before the fp32 sums.
"""
import numpy as np
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 5e-3

_REF = {}  # oracle results of the full-size fp32 inputs, shared with other dtypes' checks


def check(p, batch, variant="auto", seed=0, rows=None):
    f = inputs.factor_inputs(p, batch, seed=seed, device="cpu")
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, variant=variant, tf32=True)
    ks.sync_status()
    ref = oracle.matmul(f.X, f.values, p)
    err = oracle.max_rel_err(Y.cpu(), ref)
    assert err <= TOL, f"pattern {p} batch {batch} {variant}: err {err:.3e}"
    return err


TF32_CASES = [(1, 64, 64, 1), (1, 48, 48, 1), (2, 64, 64, 2), (1, 256, 64, 16), (1, 96, 96, 4), (4, 128, 128, 1),
              (1, 48, 48, 8), (2, 192, 48, 8), (1, 256, 256, 2), (1, 16, 16, 1), (3, 32, 16, 4), (2, 64, 64, 32),
              # c a multiple of 8 but not of 16: TF32's K step is 8
              (1, 64, 8, 1), (2, 48, 24, 2), (1, 32, 40, 4), (1, 16, 56, 8), (2, 32, 8, 16)]


@pytest.mark.parametrize("p", TF32_CASES)
@pytest.mark.parametrize("batch", [1, 67, 300])
def test_tc_kernel_tf32(p, batch):
    check(p, batch, variant="tc")


def test_tf32_products_are_tf32_on_the_tensor_cores():
    """1 + 2^-12 is not a TF32 number (10 mantissa bits): the tensor cores read
    it as 1 (by truncation or by rounding), so eight of them times 1 sum to
    exactly 8, where fp32 arithmetic gives 8 + 2^-9.  This tells the TF32 path
    from an fp32 one."""
    p = (1, 16, 8, 1)
    X = torch.full((130, 8), 1.0 + 2.0 ** -12, device=DEV)
    V = torch.ones(16 * 8, device=DEV)
    assert ks.plan(p, 130, ks.KS_TF32) == "tc"
    Y = ks.matmul(X, V, p, tf32=True)
    assert torch.equal(Y, torch.full_like(Y, 8.0))
    Yf = ks.matmul(X, V, p)  # KS_F32: fp32 FMAs
    assert torch.equal(Yf, torch.full_like(Yf, 8.0 + 2.0 ** -9))


@pytest.mark.parametrize("idx", list(range(0, 258, 3)))
def test_sweep_pattern_tf32_small_batch(idx):
    p = inputs.sweep_patterns()[idx]
    assert ks.plan(p, 67, ks.KS_TF32) == "tc"
    f = inputs.sweep_inputs(idx, batch=67)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, tf32=True)
    err = oracle.max_rel_err(Y.cpu(), oracle.matmul(f.X, f.values, p))
    assert err <= TOL, (p, err)


@pytest.mark.parametrize("name", ["vit", "gpt2"])
def test_full_size_tf32_every_row(name):
    f = getattr(inputs, name)(device=DEV)
    assert ks.plan(f.pattern, f.batch, ks.KS_TF32) == "tc"
    Y = ks.matmul(f.X, f.values, f.pattern, tf32=True)
    ks.sync_status()
    ref = oracle.matmul(f.X.cpu(), f.values.cpu(), f.pattern)
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL


@pytest.mark.parametrize("p,act", [((1, 256, 64, 16), "gelu_tanh"), ((2, 64, 64, 2), "relu"),
                                   ((1, 192, 48, 8), "gelu_erf"), ((4, 64, 32, 1), "none")])
def test_tf32_fused_bias_activation(p, act):
    f = inputs.factor_inputs(p, 257, seed=3)
    bias = torch.randn(inputs.out_features(p), generator=torch.Generator().manual_seed(6))
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, tf32=True, bias=bias.to(DEV), act=act, variant="tc")
    ks.sync_status()
    ref = oracle.matmul_epilogue(f.X, f.values, p, bias, act)
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL


def test_tf32_misaligned_output_runs_on_cuda_cores():
    """A 4-byte-aligned view is not for the tensor-core kernel; KS_TF32 then
    computes in fp32 on the CUDA cores (within the fp32 tolerance)."""
    p = (1, 64, 64, 2)
    f = inputs.factor_inputs(p, 40, seed=2)
    buf = torch.empty(40 * 128 + 1, device=DEV)
    out = buf[1:].view(40, 128)
    ks.matmul(f.X.to(DEV), f.values.to(DEV), p, tf32=True, out=out)
    ks.sync_status()
    assert oracle.max_rel_err(out.cpu(), oracle.matmul(f.X, f.values, p)) <= 1e-5
    with pytest.raises(ks.KsError):
        ks.matmul(f.X.to(DEV), f.values.to(DEV), p, tf32=True, out=out, variant="tc")


@pytest.mark.parametrize("patterns", [[(4, 64, 64, 1), (1, 64, 64, 4)], [(1, 192, 48, 8), (8, 48, 192, 1)]])
def test_tf32_two_factor_chain(patterns):
    """Two TF32 products with an fp32 intermediate: each adds at most the
    single-product error, so the chain is held to twice the TF32 tolerance."""
    c = inputs.chain_inputs(patterns, 300, seed=4)
    Y = ks.chain(c.X.to(DEV), [v.to(DEV) for v in c.factors], patterns, tf32=True)
    ks.sync_status()
    err = oracle.max_rel_err(Y.cpu(), oracle.chain(c.X, c.factors, patterns))
    assert err <= 2 * TOL, err
