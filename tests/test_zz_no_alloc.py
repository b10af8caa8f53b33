"""ks_chain_noalloc, the chain entry point that allocates no device memory.

It serves callers that must not allocate once running (their device memory
belongs to another allocator, or allocation is not allowed in their loop).
Through the C ABI it must give what ks_chain gives, call after call, although
every call reuses the library's one fixed scratch array.  Collected last on
purpose (file name), and independent of every other test.
"""
import ctypes

import pytest
import torch

import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import _lib, inputs
import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def chain_noalloc(x, factors, patterns):
    """Y through the C entry point ks_chain_noalloc on the current stream."""
    lib = _lib.load()
    n = len(factors)
    a, b, c, d = patterns[-1]
    y = torch.empty((x.shape[0], a * b * d), dtype=x.dtype, device=x.device)
    ptrs = (ctypes.c_void_p * n)(*[f.data_ptr() for f in factors])
    pats = (_lib.KsPattern * n)(*[_lib.KsPattern(*p) for p in patterns])
    st = lib.ks_chain_noalloc(x.data_ptr(), ptrs, pats, n, x.shape[0], y.data_ptr(), ks.ks_dtype_of(x),
                              torch.cuda.current_stream().cuda_stream)
    _lib.check(st)
    return y


CASES = [
    (inputs.butterfly_patterns(10), 512),                              # 1024 wide, 2 MiB intermediates
    ([(4, 64, 64, 1), (1, 64, 64, 4)], 300),                           # Monarch-like, 256 wide
    ([(1, 192, 48, 8), (8, 48, 192, 1), (1, 96, 96, 4)], 1000),       # 384 -> 1536 -> 384 -> 384
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_ks_chain_on_two_calls_in_a_row(dtype):
    for seed in (1, 2):  # two calls in a row, different inputs, same shared scratch
        for patterns, batch in CASES:
            c = inputs.chain_inputs(patterns, batch, seed=seed, dtype=dtype, device=DEV)
            y_ref = ks.chain(c.X, c.factors, patterns)
            y = chain_noalloc(c.X, c.factors, patterns)
            ks.sync_status()
            assert oracle.max_rel_err(y, y_ref) <= TOL[dtype], (patterns, seed)


def test_noalloc_largest_fitting_chain_then_rejects_one_row_more():
    pats = inputs.butterfly_patterns(12)  # 4096 fp32 = 16 KiB per row: 1024 rows fill 16 MiB
    c = inputs.chain_inputs(pats, 1024, seed=3, device=DEV, v_std=0.5 ** 0.5)
    y = chain_noalloc(c.X, c.factors, pats)
    assert oracle.max_rel_err(y, ks.chain(c.X, c.factors, pats)) <= 1e-5
    x = torch.zeros(1025, 4096, device=DEV)
    with pytest.raises(ks.KsError) as err:
        chain_noalloc(x, c.factors, pats)
    assert err.value.status == 1 and "scratch" in str(err.value)


def test_noalloc_takes_no_workspace_where_ks_matmul_would():
    """Factor (1, 256, 256, 64) at batch 256 is an fp32 product that ks_matmul
    runs with a pooled workspace (a transposed copy of its 16 MiB of values);
    its 16 MiB intermediate fits the fixed scratch exactly.  Through
    ks_chain_noalloc the library's workspace count must not move, and the
    result must still match ks_chain's."""
    pats = [(1, 256, 256, 64), (64, 16, 16, 16)]
    c = inputs.chain_inputs(pats, 256, seed=5, device=DEV)
    n0, _ = ks.workspace_info()
    ks.matmul(c.X, c.factors[0], pats[0])
    ks.sync_status()
    n1, _ = ks.workspace_info()
    assert n1 == n0 + 1  # ks_matmul took its workspace for this factor
    for _ in range(2):
        y = chain_noalloc(c.X, c.factors, pats)
        ks.sync_status()
        assert ks.workspace_info()[0] == n1
    y_ref = ks.chain(c.X, c.factors, pats)
    assert oracle.max_rel_err(y, y_ref.double()) <= 1e-5
    rows = [0, 1, 100, 255]
    ref = oracle.chain(c.X[rows].cpu(), [f.cpu() for f in c.factors], pats)
    assert oracle.max_rel_err(y[rows].cpu(), ref) <= 1e-5
