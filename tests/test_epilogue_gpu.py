"""Fused epilogue act(X K^T + bias) in every kernel family, and Monarch-style
two-factor layers through the chain, against the oracle's epilogue
(product, bias, activation in fp64).  Tolerances as for the plain product:
the epilogue runs on the fp32 accumulator before the one rounding; GELU uses
CUDA's tanhf / erff (relative error far below 1e-5)."""
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}
ACTS = ["none", "relu", "gelu_tanh", "gelu_erf"]

# (pattern, dtype, variant): each kernel family and its layouts
CASES = [((2, 4, 4, 2), torch.float32, "stream"), ((4, 2, 2, 1), torch.float32, "stream"),
         ((2, 2, 4, 8), torch.bfloat16, "stream"), ((1, 3, 5, 1), torch.float32, "stream"),
         ((2, 8, 8, 3), torch.float32, "stream"),
         ((1, 48, 48, 8), torch.float32, "fma"), ((2, 64, 64, 1), torch.float32, "fma"),
         ((1, 96, 96, 4), torch.float32, "fma"), ((2, 64, 32, 2), torch.float32, "fma"),
         ((1, 48, 48, 8), torch.bfloat16, "fma"),
         ((1, 192, 48, 8), torch.bfloat16, "tc"), ((2, 64, 64, 1), torch.bfloat16, "tc"),
         ((1, 64, 64, 2), torch.bfloat16, "tc"), ((1, 128, 64, 4), torch.bfloat16, "tc"),
         ((1, 256, 64, 16), torch.bfloat16, "tc"), ((2, 64, 32, 64), torch.bfloat16, "tc"),
         ((1, 48, 48, 16), torch.bfloat16, "tc")]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{str(c[1])[6:]}-{c[2]}")
@pytest.mark.parametrize("act", ACTS)
def test_fused_epilogue(case, act):
    p, dtype, variant = case
    batch = 131
    f = inputs.factor_inputs(p, batch, seed=sum(p), dtype=dtype)
    g = torch.Generator().manual_seed(3)
    bias = torch.randn(inputs.out_features(p), generator=g).to(dtype)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, variant=variant, bias=bias.to(DEV), act=act)
    ks.sync_status()
    ref = oracle.matmul_epilogue(f.X, f.values, p, bias, act)
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL[dtype]


@pytest.mark.parametrize("p,dtype,variant", [((1, 48, 48, 8), torch.float32, "fma"),
                                               ((2, 64, 32, 4), torch.float32, "fma"),
                                               ((1, 192, 48, 8), torch.bfloat16, "auto")])
def test_bias_not_16_byte_aligned(p, dtype, variant):
    # a bias view one element into its buffer: the fp32 kernel reads it one
    # element at a time, and the tensor-core kernel (which needs a 16-byte
    # aligned bias) is not chosen, so the CUDA-core kernel runs the product
    f = inputs.factor_inputs(p, 131, seed=9, dtype=dtype)
    g = torch.Generator().manual_seed(4)
    buf = torch.randn(inputs.out_features(p) + 1, generator=g).to(dtype).to(DEV)
    bias = buf[1:]
    assert bias.data_ptr() % 16 != 0
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, variant=variant, bias=bias, act="gelu_tanh")
    ks.sync_status()
    ref = oracle.matmul_epilogue(f.X, f.values, p, bias.cpu(), "gelu_tanh")
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL[dtype]


@pytest.mark.parametrize("act", ["relu", "gelu_erf"])
def test_activation_without_bias(act):
    p = (1, 48, 48, 8)
    f = inputs.factor_inputs(p, 77, seed=2)
    Y = ks.matmul(f.X.to(DEV), f.values.to(DEV), p, act=act)
    ks.sync_status()
    assert oracle.max_rel_err(Y.cpu(), oracle.matmul_epilogue(f.X, f.values, p, None, act)) <= 1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_monarch_mlp_layer(dtype):
    # two KS factors (Monarch-style, 256 -> 1024) then bias and GELU, one call
    pats = [(4, 64, 64, 1), (1, 256, 64, 4)]
    c = inputs.chain_inputs(pats, 300, seed=6, dtype=dtype)
    bias = torch.randn(1024, generator=torch.Generator().manual_seed(1)).to(dtype)
    Y = ks.chain(c.X.to(DEV), [v.to(DEV) for v in c.factors], pats, bias=bias.to(DEV), act="gelu_tanh")
    ks.sync_status()
    mid = oracle.matmul(c.X, c.factors[0], pats[0])
    if dtype == torch.bfloat16:  # the GPU rounds the intermediate to bf16
        mid = torch.from_numpy(mid).to(torch.bfloat16)
    ref = oracle.matmul_epilogue(mid, c.factors[1], pats[1], bias, "gelu_tanh")
    assert oracle.max_rel_err(Y.cpu(), ref) <= TOL[dtype]


def test_butterfly_chain_with_epilogue_runs_unfused():
    c = inputs.butterfly(device=DEV, batch=33, seed=2)
    bias = torch.randn(4096, device=DEV)
    Y = ks.chain(c.X, c.factors, c.patterns, bias=bias, act="relu")
    ks.sync_status()
    ref = oracle.activation(oracle.chain(c.X.cpu(), [f.cpu() for f in c.factors], c.patterns) + bias.cpu().double().numpy(), "relu")
    assert oracle.max_rel_err(Y.cpu(), ref) <= 1e-5


def test_kslinear_with_bias_gradients():
    p = (2, 32, 16, 4)
    torch.manual_seed(0)
    layer = ks.KSLinear(p, bias=True, device=DEV)
    with torch.no_grad():
        layer.bias.normal_()
    x = torch.randn(70, inputs.in_features(p), device=DEV, requires_grad=True)
    y = layer(x)
    g = torch.randn_like(y)
    y.backward(g)
    ks.sync_status()
    ref = oracle.matmul_epilogue(x.detach().cpu(), layer.values.detach().cpu(), p, layer.bias.detach().cpu(), "none")
    assert oracle.max_rel_err(y.detach().cpu(), ref) <= 1e-5
    assert oracle.max_rel_err(layer.bias.grad.cpu(), g.cpu().double().sum(0).numpy()) <= 1e-5


def test_epilogue_argument_errors():
    p = (1, 8, 8, 1)
    x = torch.zeros(4, 8, device=DEV)
    v = torch.zeros(64, device=DEV)
    with pytest.raises(ValueError):
        ks.matmul(x, v, p, act="swish")
    with pytest.raises(ValueError):
        ks.matmul(x, v, p, bias=torch.zeros(7, device=DEV))
    out = torch.zeros(4, 8, device=DEV)
    with pytest.raises(ks.KsError) as e:  # bias inside Y
        ks.matmul(x, v, p, out=out, bias=out[0])
    assert e.value.status == 1
