"""Parity of the CUDA kernels with the CPU oracle, element by element on the
same seeded inputs, through the C ABI.

Tolerance (max|Y - Y_ref| / max|Y_ref|): 1e-5 for fp32 (CUDA-core FMA),
5e-3 for TF32, 1e-2 for BF16 (bf16 output rounding dominates).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, "tf32": 5e-3, torch.bfloat16: 1e-2}
DEV = "cuda"


def run_and_check(p, batch, dtype=torch.float32, variant="auto", seed=0, x_dist="normal", tf32=False,
                  rows=None):
    f = inputs.factor_inputs(p, batch, seed=seed, dtype=dtype, device="cpu", x_dist=x_dist)
    X, V = f.X.to(DEV), f.values.to(DEV)
    Y = ks.matmul(X, V, p, variant=variant, tf32=tf32)
    ks.sync_status()
    assert Y.shape == (batch, inputs.out_features(p))
    if rows is None:
        ref = oracle.matmul(f.X, f.values, p)
        got = Y.cpu()
    else:
        ref = oracle.matmul(f.X[rows], f.values, p)
        got = Y[rows].cpu()
    err = oracle.max_rel_err(got, ref)
    tol = TOL["tf32"] if tf32 else TOL[dtype]
    assert err <= tol, f"pattern {p} batch {batch} {dtype} {variant}: err {err:.3e} > {tol}"
    return err


TINY = [(2, 4, 4, 2), (1, 3, 5, 1), (3, 2, 2, 3), (2, 1, 1, 4), (1, 8, 8, 8), (4, 2, 2, 1), (5, 3, 7, 2)]


@pytest.mark.parametrize("p", TINY)
@pytest.mark.parametrize("batch", [1, 7, 33])
def test_stream_kernel_tiny(p, batch):
    run_and_check(p, batch, variant="stream")


def test_toy_config():
    t = inputs.toy()
    Y = ks.matmul(t.X.to(DEV), t.values.to(DEV), t.pattern)
    err = oracle.max_rel_err(Y.cpu(), oracle.matmul(t.X, t.values, t.pattern))
    assert err <= 1e-5


FMA_CASES = [
    (1, 48, 48, 8), (1, 64, 64, 1), (2, 64, 64, 2), (1, 96, 96, 4), (1, 192, 48, 8), (1, 256, 64, 16),
    (2, 128, 128, 8), (4, 48, 48, 1), (1, 16, 16, 1), (1, 24, 8, 1), (3, 40, 12, 4), (2, 20, 36, 2),
    (1, 48, 48, 32), (8, 192, 192, 1), (1, 256, 256, 2), (2, 9, 12, 12),
]


@pytest.mark.parametrize("p", FMA_CASES)
@pytest.mark.parametrize("batch", [1, 63, 130])
def test_fma_kernel(p, batch):
    run_and_check(p, batch, variant="fma")


@pytest.mark.parametrize("p", [(1, 48, 48, 8), (1, 64, 64, 16), (2, 64, 64, 1), (1, 96, 96, 4), (1, 8, 16, 2)])
def test_fma_kernel_bf16(p):
    run_and_check(p, 70, dtype=torch.bfloat16, variant="fma")


# Block shapes (b, c) in {1, 2, 4}^2 take the register-weight streaming kernel:
# d a multiple of the 16-byte element count (l-vector layout), or d in
# {1, 2} (and 4 for bf16) with whole blocks merged into 16-byte runs; a
# includes values the merged unit does not divide (those fall back).
STREAM_REG = [(a, b, c, d) for (b, c) in [(1, 1), (1, 2), (2, 1), (2, 2), (2, 4), (4, 2), (4, 4), (1, 4)]
              for (a, d) in [(8, 1), (4, 2), (2, 4), (2, 8), (3, 1), (1, 16), (6, 2)]]


@pytest.mark.parametrize("p", STREAM_REG)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_stream_register_kernel_layouts(p, dtype):
    for batch in (1, 7, 300):
        run_and_check(p, batch, dtype=dtype, variant="stream")


@pytest.mark.parametrize("p", [(2, 2, 2, 8), (4, 8, 8, 4), (1, 3, 3, 16), (2, 4, 4, 1)])
def test_stream_kernel_bf16(p):
    run_and_check(p, 37, dtype=torch.bfloat16, variant="stream")


@pytest.mark.parametrize("p", [(1, 192, 48, 8), (2, 64, 64, 2)])
def test_tf32_dtype_runs_on_the_tensor_cores(p):
    assert ks.plan(p, 100, ks.KS_TF32) == "tc"
    run_and_check(p, 100, tf32=True)


def test_auto_on_odd_pattern_uses_catch_all():
    assert ks.plan((3, 5, 7, 3), 10) == "stream"
    run_and_check((3, 5, 7, 3), 10)


def test_misaligned_views_take_the_scalar_path():
    p = (1, 48, 48, 8)
    f = inputs.factor_inputs(p, 20)
    Xbuf = torch.zeros(20 * 384 + 1, device=DEV)
    Xbuf[1:] = f.X.reshape(-1).to(DEV)
    X = Xbuf[1:].view(20, 384)  # 4-byte aligned, not 16
    Y = ks.matmul(X, f.values.to(DEV), p)
    assert oracle.max_rel_err(Y.cpu(), oracle.matmul(f.X, f.values, p)) <= 1e-5
    with pytest.raises(ks.KsError):
        ks.matmul(X, f.values.to(DEV), p, variant="fma")


def test_empty_batch():
    X = torch.zeros(0, 384, device=DEV)
    V = torch.zeros(192 * 48 * 8, device=DEV)
    assert ks.matmul(X, V, (1, 192, 48, 8)).shape == (0, 1536)


def test_special_cases_dense_and_diagonal():
    # a = d = 1: a dense GEMM; b = c = 1: diagonal scaling
    f = inputs.factor_inputs((1, 64, 32, 1), 50)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), (1, 64, 32, 1)).cpu().double()
    ref = f.X.double() @ f.values.reshape(64, 32).double().T
    assert oracle.max_rel_err(Y, ref) <= 1e-5
    g = inputs.factor_inputs((6, 1, 1, 4), 9)
    Y = ks.matmul(g.X.to(DEV), g.values.to(DEV), (6, 1, 1, 4)).cpu()
    assert torch.equal(Y, g.X * g.values.reshape(1, 24))


@pytest.mark.parametrize("idx", list(range(0, 258, 1)))
def test_sweep_pattern_fp32_small_batch(idx):
    p = inputs.sweep_patterns()[idx]
    f = inputs.sweep_inputs(idx, batch=67)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p)
    err = oracle.max_rel_err(Y.cpu(), oracle.matmul(f.X, f.values, p))
    assert err <= 1e-5, (p, err)


@pytest.mark.parametrize("idx", list(range(0, 258, 3)))
def test_sweep_pattern_bf16_small_batch(idx):
    p = inputs.sweep_patterns()[idx]
    f = inputs.sweep_inputs(idx, batch=67, dtype=torch.bfloat16)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p)
    err = oracle.max_rel_err(Y.cpu(), oracle.matmul(f.X, f.values, p))
    assert err <= 1e-2, (p, err)


def sampled_rows(batch, k=48, seed=1):
    g = np.random.default_rng(seed)
    rows = set(g.choice(batch, size=min(k, batch), replace=False).tolist())
    rows |= {0, batch - 1}
    return sorted(rows)


@pytest.mark.parametrize("name,dtype", [("vit", torch.float32), ("gpt2", torch.float32), ("gpt2", torch.bfloat16)])
def test_full_size_configs_every_row(name, dtype):
    f = getattr(inputs, name)(dtype=dtype, device=DEV)
    Y = ks.matmul(f.X, f.values, f.pattern)
    ks.sync_status()
    ref = oracle.matmul(f.X.cpu(), f.values.cpu(), f.pattern)
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL[dtype]


@pytest.mark.parametrize("idx", [0, 38, 77, 120, 150, 200, 229, 257])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_full_size_sweep_patterns_sampled_rows(idx, dtype):
    p = inputs.sweep_patterns()[idx]
    f = inputs.sweep_inputs(idx, dtype=dtype, device=DEV)
    Y = ks.matmul(f.X, f.values, p)
    rows = sampled_rows(f.batch, k=24)
    ref = oracle.matmul(f.X[rows].cpu(), f.values.cpu(), p)
    assert oracle.max_rel_err(Y[rows].cpu(), ref) <= TOL[dtype]


# Full-size sweep patterns compared on every row: the tensor-core kernel's l
# widths 1 (48 and 256 x 64 blocks, a = 64 and 8), 2, 4, 8 with d = 8 (whole
# 256-byte rows) and 8 with d >= 16 (four-dimensional boxes), the last with
# several k passes per X tile (b = 96, 128 with d = 16, 32); in bf16, 16 l with
# d = 16 and b = 48 (whole 512-byte rows, passes of 16 k, contiguous output
# boxes) and with d = 64 (four-dimensional boxes both ways, six passes); the
# fp32 kernel's l widths 1, 2, 4, 8 (d >= 16 with the transposed-values
# workspace).
FULL_ROWS = [82, 205, 127, 48, 248, 117, 36, 234, 4, 208]


@pytest.mark.parametrize("idx", FULL_ROWS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_full_size_sweep_patterns_every_row(idx, dtype):
    p = inputs.sweep_patterns()[idx]
    f = inputs.sweep_inputs(idx, dtype=dtype, device=DEV)
    Y = ks.matmul(f.X, f.values, p)
    ks.sync_status()
    ref = oracle.matmul(f.X.cpu(), f.values.cpu(), p)
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL[dtype], p


TC_CASES = [(1, 64, 64, 1), (1, 48, 48, 1), (2, 64, 64, 2), (1, 256, 64, 16), (1, 96, 96, 4), (4, 128, 128, 1),
            (1, 48, 48, 8), (2, 192, 48, 8), (1, 256, 256, 2), (1, 16, 16, 1), (3, 32, 16, 4), (2, 64, 64, 32),
            # bf16 with 16 l per tile: passes of 16 k (double-buffered), d = 64, one chunk of j
            (1, 48, 48, 16), (2, 96, 64, 64), (1, 32, 16, 64)]


@pytest.mark.parametrize("p", TC_CASES)
@pytest.mark.parametrize("batch", [1, 67, 300])
def test_tc_kernel_bf16(p, batch):
    run_and_check(p, batch, dtype=torch.bfloat16, variant="tc")


def test_tc_rejects_fp32_and_unsupported():
    f = inputs.factor_inputs((1, 64, 64, 1), 8)
    with pytest.raises(ks.KsError):
        ks.matmul(f.X.to(DEV), f.values.to(DEV), (1, 64, 64, 1), variant="tc")
    g = inputs.factor_inputs((1, 64, 40, 1), 8, dtype=torch.bfloat16)  # c not a multiple of 16
    with pytest.raises(ks.KsError):
        ks.matmul(g.X.to(DEV), g.values.to(DEV), (1, 64, 40, 1), variant="tc")
