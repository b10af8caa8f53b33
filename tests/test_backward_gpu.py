"""Gradients of Y = X K^T on the GPU (ks_matmul_dx, ks_matmul_dv and the
KSLinear layer built on them) against the oracle's dx / dv, element by element
on the same seeded inputs.

Tolerances (max|G - G_ref| / max|G_ref|): dX as a forward product, 1e-5 fp32 and
1e-2 bf16.  dV sums over the whole batch in fp32 (row ranges summed in order,
then the ranges): 1e-5 up to a few hundred rows, 1e-4 at the full ViT batch of
25216 rows (the fp32 error of such a sum grows like its length times the unit
roundoff in the worst case, ~25216 x 6e-8 = 1.5e-3, and like its square root in
practice); bf16 inputs are exact in fp32, so bf16 dV only adds its final
rounding, 1e-2.
"""
import pytest
import torch

import oracle
import kronecker_sparse_matrix_b200 as ks
from kronecker_sparse_matrix_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}

PATTERNS = [(2, 4, 4, 2), (1, 3, 5, 1), (3, 2, 7, 3), (1, 48, 48, 8), (2, 64, 32, 4), (1, 96, 80, 1),
            (4, 16, 24, 2), (1, 192, 48, 8), (2, 20, 36, 16), (1, 130, 70, 6), (8, 4, 4, 1)]


def grad_inputs(p, batch, dtype, seed):
    f = inputs.factor_inputs(p, batch, seed=seed, dtype=dtype, device="cpu")
    g = torch.Generator().manual_seed(seed + 77)
    dy = torch.randn(batch, inputs.out_features(p), generator=g).to(dtype)
    return f.X, f.values, dy


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dx_matches_oracle(p, dtype):
    for batch in (1, 37, 300):
        X, V, dy = grad_inputs(p, batch, dtype, seed=sum(p) + batch)
        dx = ks.matmul_dx(dy.to(DEV), V.to(DEV), p)
        ks.sync_status()
        assert dx.shape == (batch, inputs.in_features(p))
        assert oracle.max_rel_err(dx.cpu(), oracle.dx(dy, V, p)) <= TOL[dtype], (p, batch)


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dv_matches_oracle(p, dtype):
    for batch in (1, 9, 300, 1111):
        X, V, dy = grad_inputs(p, batch, dtype, seed=sum(p) + 3 * batch)
        dv = ks.matmul_dv(dy.to(DEV), X.to(DEV), p)
        ks.sync_status()
        assert dv.shape == (p[0], p[3], p[1], p[2])
        assert oracle.max_rel_err(dv.cpu().reshape(-1), oracle.dv(dy, X, p)) <= TOL[dtype], (p, batch)


# bf16 patterns that take the tensor-core dV kernel (d % 8 == 0, c % 16 == 0 up to
# 64, b >= 128): one and several 128-k tiles (b = 160: a tail of 32 k), one and
# three groups of 8 l, several blocks, c = 16 .. 64.
DV_TC_PATTERNS = [(1, 256, 64, 16), (2, 128, 32, 8), (1, 160, 16, 24), (3, 128, 64, 8), (1, 192, 48, 8)]


def cuda_kernel_names(fn):
    with torch.profiler.profile(activities=[torch.profiler.ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return {e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA}


@pytest.mark.parametrize("p", DV_TC_PATTERNS)
def test_dv_tensor_core_path_matches_oracle(p):
    for batch in (1, 9, 300, 1111):
        X, V, dy = grad_inputs(p, batch, torch.bfloat16, seed=sum(p) + 5 * batch)
        dv = ks.matmul_dv(dy.to(DEV), X.to(DEV), p)
        ks.sync_status()
        assert oracle.max_rel_err(dv.cpu().reshape(-1), oracle.dv(dy, X, p)) <= TOL[torch.bfloat16], (p, batch)


def test_dv_tensor_core_path_full_gpt2_batch():
    f = inputs.gpt2(dtype=torch.bfloat16, device=DEV)
    p = f.pattern
    g = torch.Generator(device=DEV).manual_seed(6)
    dy = torch.randn(f.batch, inputs.out_features(p), generator=g, device=DEV).to(torch.bfloat16)
    names = cuda_kernel_names(lambda: ks.matmul_dv(dy, f.X, p))
    assert any("dv_tc_kernel" in n for n in names), names
    dv = ks.matmul_dv(dy, f.X, p)
    ks.sync_status()
    assert oracle.max_rel_err(dv.cpu().reshape(-1), oracle.dv(dy.cpu(), f.X.cpu(), p)) <= TOL[torch.bfloat16]


def test_dv_full_vit_batch():
    f = inputs.vit(device=DEV)
    p = f.pattern
    g = torch.Generator(device=DEV).manual_seed(5)
    dy = torch.randn(f.batch, inputs.out_features(p), generator=g, device=DEV)
    dv = ks.matmul_dv(dy, f.X, p)
    ks.sync_status()
    assert oracle.max_rel_err(dv.cpu().reshape(-1), oracle.dv(dy.cpu(), f.X.cpu(), p)) <= 1e-4


def test_dv_of_empty_batch_is_zero():
    p = (2, 8, 4, 2)
    out = torch.full((2, 2, 8, 4), 7.0, device=DEV)
    ks.matmul_dv(torch.empty(0, 32, device=DEV), torch.empty(0, 16, device=DEV), p, out=out)
    ks.sync_status()
    assert torch.count_nonzero(out).item() == 0


def test_dv_is_deterministic():
    p = (1, 64, 64, 8)
    X, V, dy = grad_inputs(p, 5000, torch.float32, seed=1)
    dy, X = dy.to(DEV), X.to(DEV)
    a = ks.matmul_dv(dy, X, p)
    b = ks.matmul_dv(dy, X, p)
    ks.sync_status()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_kslinear_layer_gradients(dtype):
    p = (2, 32, 16, 4)
    torch.manual_seed(0)
    layer = ks.KSLinear(p, dtype=dtype, device=DEV)
    x = torch.randn(3, 50, inputs.in_features(p), device=DEV).to(dtype).requires_grad_(True)
    y = layer(x)
    g = torch.randn_like(y)
    y.backward(g)
    ks.sync_status()
    V = layer.values.detach().cpu()
    X2 = x.detach().cpu().reshape(-1, inputs.in_features(p))
    G2 = g.cpu().reshape(-1, inputs.out_features(p))
    assert oracle.max_rel_err(y.detach().cpu().reshape(-1, inputs.out_features(p)), oracle.matmul(X2, V, p)) <= TOL[dtype]
    assert oracle.max_rel_err(x.grad.cpu().reshape(-1, inputs.in_features(p)), oracle.dx(G2, V, p)) <= TOL[dtype]
    assert oracle.max_rel_err(layer.values.grad.cpu().reshape(-1), oracle.dv(G2, X2, p)) <= TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("batch,width", [(1, 1), (63, 300), (1000, 1536), (25216, 384), (5, 4097)])
def test_bias_grad_matches_oracle(dtype, batch, width):
    g = torch.Generator().manual_seed(batch + width)
    dy = torch.randn(batch, width, generator=g).to(dtype)
    db = ks.bias_grad(dy.to(DEV))
    ks.sync_status()
    tol = 1e-5 if dtype == torch.float32 else 1e-2
    assert oracle.max_rel_err(db.cpu(), oracle.bias_grad(dy)) <= tol


def test_bias_grad_of_empty_batch_is_zero_and_deterministic():
    z = ks.bias_grad(torch.zeros(0, 77, device=DEV))
    assert torch.equal(z.cpu(), torch.zeros(77))
    dy = torch.randn(9000, 1536, device=DEV)
    assert torch.equal(ks.bias_grad(dy), ks.bias_grad(dy))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_kslinear_bias_gradient_runs_in_the_library(dtype):
    p = (1, 64, 32, 4)
    torch.manual_seed(2)
    layer = ks.KSLinear(p, bias=True, dtype=dtype, device=DEV)
    x = torch.randn(130, inputs.in_features(p), device=DEV).to(dtype)
    y = layer(x)
    g = torch.randn_like(y)
    y.backward(g)
    ks.sync_status()
    tol = 1e-5 if dtype == torch.float32 else 1e-2
    assert oracle.max_rel_err(layer.bias.grad.cpu(), oracle.bias_grad(g.cpu())) <= tol


def test_kslinear_trains_toward_a_ks_target():
    # a few SGD steps on a realisable target must reduce the loss (a smoke test
    # of the whole training step on the GPU path)
    p = (4, 16, 16, 2)
    torch.manual_seed(1)
    target = ks.KSLinear(p, device=DEV)
    layer = ks.KSLinear(p, device=DEV)
    opt = torch.optim.SGD(layer.parameters(), lr=2.0)  # mean over 64 outputs scales the gradient by 1/32
    x = torch.randn(512, inputs.in_features(p), device=DEV)
    with torch.no_grad():
        y_t = target(x)
    losses = []
    for _ in range(30):
        opt.zero_grad()
        loss = ((layer(x) - y_t) ** 2).mean()
        loss.backward()
        opt.step()
        losses.append(loss.item())
    assert losses[-1] < 0.5 * losses[0]


def test_gradient_argument_errors():
    p = (2, 4, 4, 2)  # in = out = 16 features, 64 values
    buf = torch.zeros(200, device=DEV)
    x = buf[:48].view(3, 16)
    dy = torch.zeros(3, 16, device=DEV)
    with pytest.raises(ks.KsError) as e:
        ks.matmul_dv(dy, x, p, out=buf[40:104].view(2, 2, 4, 4))  # dV overlaps X
    assert e.value.status == 1
    with pytest.raises(ks.KsError) as e:
        ks.matmul_dx(dy, torch.zeros(64, device=DEV), p, out=dy)  # dX overlaps dY
    assert e.value.status == 1
