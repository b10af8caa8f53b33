"""Every tile of the fp32 CUDA-core kernel (ks_fma32.cu), against the oracle.

The kernel picks one of 19 tiles (l width DL x rows x k) from the pattern and
the batch.  Each case below is a small product for which the library's tile
choice lands on a different one of them, with a batch that is not a multiple
of the tile's rows, k not a multiple of the tile's k where the tile allows it,
and c = 12 (a partial last stage of 8 j).  Full-batch cases with d % 8 == 0
take the path that stages a transposed copy of the values; those are checked
on sampled rows.  Tolerance: 1e-5 (max|Y - Y_ref| / max|Y_ref|).
"""
import numpy as np
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (pattern, batch) -> the tile it selects (DL, rows x k)
TILE_CASES = [
    ((3, 52, 12, 16), 1023),   # 8, 64 x 64
    ((16, 32, 12, 16), 511),   # 8, 128 x 32
    ((1, 12, 12, 8), 63),      # 8, 64 x 48
    ((37, 12, 12, 16), 130),   # 8, 128 x 24
    ((37, 52, 12, 4), 257),    # 4, 128 x 64
    ((1, 200, 12, 4), 4099),   # 4, 64 x 128
    ((2, 12, 12, 4), 16385),   # 4, 256 x 32
    ((37, 12, 12, 4), 257),    # 4, 128 x 48
    ((1, 12, 12, 4), 63),      # 4, 64 x 96
    ((37, 100, 12, 2), 257),   # 2, 128 x 128
    ((2, 52, 12, 2), 16385),   # 2, 256 x 64
    ((16, 12, 12, 2), 4099),   # 2, 512 x 32
    ((1, 12, 12, 2), 63),      # 2, 128 x 96
    ((2, 12, 12, 2), 16385),   # 2, 256 x 48
    ((37, 200, 12, 1), 257),   # 1, 256 x 128
    ((8, 52, 12, 1), 8191),    # 1, 512 x 64
    ((5, 200, 12, 1), 4099),   # 1, 128 x 256
    ((1, 12, 12, 1), 63),      # 1, 256 x 96
    ((8, 12, 12, 1), 8191),    # 1, 512 x 48
]


@pytest.mark.parametrize("p,batch", TILE_CASES)
def test_every_fp32_tile(p, batch):
    f = inputs.factor_inputs(p, batch, seed=sum(p) + batch)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p)
    ks.sync_status()
    err = oracle.max_rel_err(Y.cpu(), oracle.matmul(f.X, f.values, p))
    assert err <= 1e-5, (p, batch, err)


# one case per l width with the fused bias and GELU (the epilogue's second copy)
@pytest.mark.parametrize("p,batch", [TILE_CASES[0], TILE_CASES[4], TILE_CASES[9], TILE_CASES[14]])
def test_fp32_tiles_with_fused_epilogue(p, batch):
    f = inputs.factor_inputs(p, batch, seed=7 + batch)
    bias = torch.randn(inputs.out_features(p), generator=torch.Generator().manual_seed(batch))
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, bias=bias.to(DEV), act="gelu_tanh")
    ks.sync_status()
    ref = oracle.matmul_epilogue(f.X, f.values, p, bias, "gelu_tanh")
    assert oracle.max_rel_err(Y.cpu(), ref) <= 1e-5


# full batch, d % 8 == 0, >= 2^30 flop: values staged from a transposed copy
@pytest.mark.parametrize("p", [(16, 32, 12, 16), (37, 12, 12, 16), (3, 52, 12, 16)])
def test_fp32_tiles_transposed_values_full_batch(p):
    batch = inputs.SWEEP_BATCH
    f = inputs.factor_inputs(p, batch, seed=11, device=DEV)
    Y = ks.matmul(f.X, f.values, p)
    ks.sync_status()
    g = np.random.default_rng(3)
    rows = sorted(set(g.choice(batch, size=24, replace=False).tolist()) | {0, batch - 1})
    ref = oracle.matmul(f.X[rows].cpu(), f.values.cpu(), p)
    assert oracle.max_rel_err(Y[rows].cpu(), ref) <= 1e-5
