"""ks_matmul_host: a batch in host memory streamed through the GPU in chunks
(copies overlapping the products), against the oracle and against ks_matmul on
the same rows already on the device."""
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: 1e-5, "tf32": 5e-3, torch.bfloat16: 1e-2}


def host_inputs(p, batch, dtype=torch.float32, seed=0, pinned=True):
    f = inputs.factor_inputs(p, batch, seed=seed, dtype=dtype)
    X, V = f.X, f.values
    if pinned:
        X, V = X.pin_memory(), V.pin_memory()
    return f, X, V


@pytest.mark.parametrize("p,batch", [((1, 192, 48, 8), 5000), ((2, 64, 64, 2), 777), ((1, 256, 64, 16), 8192),
                                     ((4, 2, 2, 8), 3000), ((3, 5, 7, 3), 1500)])
def test_host_product_matches_oracle_and_device_path(p, batch):
    f, X, V = host_inputs(p, batch)
    Y = ks.matmul_host(X, V, p)
    torch.cuda.current_stream().synchronize()
    ks.sync_status()
    assert oracle.max_rel_err(Y, oracle.matmul(f.X, f.values, p)) <= 1e-5
    # fp32 FMAs in j order whatever the chunking: equal to the device-resident product
    Yd = ks.matmul(X.to(DEV), V.to(DEV), p)
    assert torch.equal(Y, Yd.cpu())


@pytest.mark.parametrize("dtype,tf32", [(torch.bfloat16, False), (torch.float32, True)])
def test_host_product_tensor_core_dtypes(dtype, tf32):
    p = (1, 256, 64, 16)
    f, X, V = host_inputs(p, 6000, dtype=dtype, seed=3)
    Y = ks.matmul_host(X, V, p, tf32=tf32)
    torch.cuda.current_stream().synchronize()
    ks.sync_status()
    assert oracle.max_rel_err(Y, oracle.matmul(f.X, f.values, p)) <= TOL["tf32" if tf32 else dtype]


def test_host_product_pageable_memory_and_empty_batch():
    p = (2, 48, 48, 4)
    f, X, V = host_inputs(p, 2500, seed=5, pinned=False)
    Y = ks.matmul_host(X, V, p)
    torch.cuda.current_stream().synchronize()
    assert oracle.max_rel_err(Y, oracle.matmul(f.X, f.values, p)) <= 1e-5
    E = ks.matmul_host(torch.zeros(0, 384), V, p)
    assert E.shape == (0, 2 * 48 * 4)


def test_host_product_is_ordered_on_the_callers_stream():
    # the call waits for earlier work on the stream and the stream waits for it
    p = (1, 64, 64, 4)
    f, X, V = host_inputs(p, 4096, seed=7)
    s = torch.cuda.Stream()
    out = torch.empty(4096, 256, pin_memory=True)
    with torch.cuda.stream(s):
        torch.cuda._sleep(1000000)  # about a millisecond of earlier work on s
        ks.matmul_host(X, V, p, out=out, stream=s)
    s.synchronize()
    assert oracle.max_rel_err(out, oracle.matmul(f.X, f.values, p)) <= 1e-5
