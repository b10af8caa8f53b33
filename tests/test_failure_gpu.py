"""Failure detection without a GPU fault.

KS_FAULT_INJECT=alloc makes every workspace allocation fail on the host: each
entry point that needs a workspace returns KS_ERR_ALLOC before it launches
anything, so its output is left as it was; ks_matmul, whose fp32 workspace is
optional, reads the values in place and is still correct.

KS_FAULT_INJECT=timeout makes the tensor-core kernels' pipeline waits give up
at once (the forward product and the bf16 values gradient): the kernel
abandons its loop, drains its in-flight copies and MMAs (bounded), frees its
tensor memory and returns, and ks_sync_status reports KS_ERR_TIMEOUT.  The
context stays usable: the next call on the same stream is checked against the
oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENTINEL = 7.0


def sentinel_like(shape, dtype=torch.float32):
    return torch.full(shape, SENTINEL, dtype=dtype, device=DEV)


def expect_alloc_failure(fn):
    with pytest.raises(ks.KsError) as err:
        fn()
    assert err.value.status == 4 and "workspace" in str(err.value)


def test_injected_allocation_failures_leave_outputs_untouched(monkeypatch):
    pats = [(4, 64, 64, 1), (1, 64, 64, 4)]
    c = inputs.chain_inputs(pats, 200, seed=11, device=DEV)
    p = (2, 64, 32, 4)
    f = inputs.factor_inputs(p, 150, seed=12, device=DEV)
    dy = torch.randn(150, inputs.out_features(p), generator=torch.Generator(device=DEV).manual_seed(13), device=DEV)
    bf = inputs.butterfly(batch=1, log2n=6, seed=14)
    A = torch.tensor(np.ascontiguousarray(oracle.chain(np.eye(64), bf.factors, bf.patterns).T), dtype=torch.float32,
                     device=DEV)

    y = sentinel_like((200, 256))
    dx = sentinel_like((150, inputs.in_features(p)))
    dv = sentinel_like((2, 4, 64, 32))
    facs = [sentinel_like((q[0] * q[1] * q[2] * q[3],)) for q in inputs.butterfly_patterns(6)]
    monkeypatch.setenv("KS_FAULT_INJECT", "alloc")
    expect_alloc_failure(lambda: ks.chain(c.X, c.factors, pats, out=y))
    expect_alloc_failure(lambda: ks.matmul_dx(dy, f.values, p, out=dx))
    expect_alloc_failure(lambda: ks.matmul_dv(dy, f.X, p, out=dv))

    def factorize():
        import ctypes
        from kronecker_sparse_matrix_b200 import _lib
        ptrs = (ctypes.c_void_p * 6)(*[t.data_ptr() for t in facs])
        _lib.check(_lib.load().ks_butterfly_factorize(A.data_ptr(), 6, ptrs, ks.KS_F32,
                                                      torch.cuda.current_stream().cuda_stream))
    expect_alloc_failure(factorize)
    ks.sync_status()
    for t in [y, dx, dv] + facs:
        assert bool((t == SENTINEL).all())

    monkeypatch.delenv("KS_FAULT_INJECT")
    ks.chain(c.X, c.factors, pats, out=y)
    ks.matmul_dx(dy, f.values, p, out=dx)
    ks.matmul_dv(dy, f.X, p, out=dv)
    ks.sync_status()
    assert oracle.max_rel_err(y.cpu(), oracle.chain(c.X.cpu(), [v.cpu() for v in c.factors], pats)) <= 1e-5
    assert oracle.max_rel_err(dx.cpu(), oracle.dx(dy.cpu(), f.values.cpu(), p)) <= 1e-5
    assert oracle.max_rel_err(dv.cpu().reshape(-1), oracle.dv(dy.cpu(), f.X.cpu(), p)) <= 1e-5


def test_matmul_reads_values_in_place_when_its_workspace_fails(monkeypatch):
    # fp32, d % 8 == 0, b % 4 == 0, >= 2^30 flop: this product normally stages a
    # transposed copy of the values in a pooled workspace
    p = (1, 128, 128, 16)
    f = inputs.factor_inputs(p, 2048, seed=15, device=DEV)
    before, _ = ks.workspace_info()
    Y0 = ks.matmul(f.X, f.values, p)
    ks.sync_status()
    assert ks.workspace_info()[0] == before + 1
    monkeypatch.setenv("KS_FAULT_INJECT", "alloc")
    Y1 = ks.matmul(f.X, f.values, p)
    ks.sync_status()
    assert ks.workspace_info()[0] == before + 1
    assert oracle.max_rel_err(Y1, Y0.double()) <= 1e-6  # the same fp32 FMAs, whichever copy of the values
    rows = [0, 1, 777, 2047]
    assert oracle.max_rel_err(Y1[rows].cpu(), oracle.matmul(f.X[rows].cpu(), f.values.cpu(), p)) <= 1e-5


@pytest.mark.parametrize("p,dtype,tf32", [((1, 64, 64, 1), torch.bfloat16, False),
                                          ((2, 64, 64, 2), torch.float32, True),
                                          ((1, 64, 64, 16), torch.bfloat16, False)])
def test_tc_wait_timeout_is_reported_and_the_next_call_is_correct(monkeypatch, p, dtype, tf32):
    f = inputs.factor_inputs(p, 300, seed=16, dtype=dtype, device=DEV)
    dt = ks.ks_dtype_of(f.X, tf32)
    assert ks.plan(p, 300, dt) == "tc"
    ks.sync_status()  # nothing pending before the injected failure
    monkeypatch.setenv("KS_FAULT_INJECT", "timeout")
    Y = ks.matmul(f.X, f.values, p, tf32=tf32)  # the launch itself succeeds
    with pytest.raises(ks.KsError) as err:
        ks.sync_status()
    assert err.value.status == 6
    ks.sync_status()  # the status word was cleared by the report
    monkeypatch.delenv("KS_FAULT_INJECT")
    Y = ks.matmul(f.X, f.values, p, tf32=tf32)
    ks.sync_status()
    tol = 5e-3 if tf32 else 1e-2
    assert oracle.max_rel_err(Y.cpu(), oracle.matmul(f.X.cpu(), f.values.cpu(), p)) <= tol


def test_dv_tensor_core_wait_timeout_is_reported_and_the_next_call_is_correct(monkeypatch):
    p = (1, 256, 64, 16)  # bf16 dV on the tensor cores
    f = inputs.factor_inputs(p, 300, seed=17, dtype=torch.bfloat16, device=DEV)
    dy = torch.randn(300, inputs.out_features(p), generator=torch.Generator(device=DEV).manual_seed(18),
                     device=DEV).to(torch.bfloat16)
    ks.sync_status()
    monkeypatch.setenv("KS_FAULT_INJECT", "timeout")
    ks.matmul_dv(dy, f.X, p)  # the launches themselves succeed
    with pytest.raises(ks.KsError) as err:
        ks.sync_status()
    assert err.value.status == 6
    ks.sync_status()
    monkeypatch.delenv("KS_FAULT_INJECT")
    dv = ks.matmul_dv(dy, f.X, p)
    ks.sync_status()
    assert oracle.max_rel_err(dv.cpu().reshape(-1), oracle.dv(dy.cpu(), f.X.cpu(), p)) <= 1e-2
