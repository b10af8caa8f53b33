"""B200 (sm_100a) library for multiplication by Kronecker-sparse (KS) matrices.

Y = X K^T with K of pattern (a, b, c, d), support I_a (x) 1_{b x c} (x) I_d
and values[a][d][b][c], for one factor (``matmul``) or a chain of factors
(``chain``) -- the operation of the taxoreview.com page on Kronecker-sparse
matrix multiplication (first abstract).  Every step runs in the CUDA kernels
of ``libks_b200.so`` behind the C ABI of ``include/ks.h``; this module only
marshals torch tensors (device memory and streams) into that ABI.  There is no
CPU or PyTorch fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import (KS_BF16, KS_F32, KS_TF32, KS_VARIANT_AUTO, KS_VARIANT_FMA,  # noqa: F401
                   KS_CHAIN_UNFUSED, KS_VARIANT_STREAM, KS_VARIANT_TC, KsError, KsPattern, VARIANTS)

Pattern = Tuple[int, int, int, int]

__all__ = ["matmul", "matmul_host", "matmul_dx", "matmul_dv", "bias_grad", "chain", "butterfly_factorize", "KSLinear",
           "plan", "sync_status", "workspace_info", "ks_dtype_of", "KsError", "VARIANTS"]


def ks_dtype_of(t: torch.Tensor, tf32: bool = False) -> int:
    if t.dtype == torch.float32:
        return KS_TF32 if tf32 else KS_F32
    if t.dtype == torch.bfloat16:
        if tf32:
            raise ValueError("tf32 applies to fp32 tensors only")
        return KS_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")


def _stream_ptr(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(s.cuda_stream)


def _variant(v) -> int:
    if isinstance(v, str):
        return VARIANTS[v]
    return int(v)


def matmul(x: torch.Tensor, values: torch.Tensor, pattern: Pattern, *, out: Optional[torch.Tensor] = None,
           tf32: bool = False, variant="auto", bias: Optional[torch.Tensor] = None, act: str = "none",
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Y = act(X K^T + bias) for one KS factor.  x: (batch, a*c*d) CUDA tensor
    (fp32 or bf16), values: a*b*c*d entries in [a][d][b][c] order, same
    dtype/device; bias: a*b*d entries or None; act: "none", "relu",
    "gelu_tanh" or "gelu_erf" (fused into the kernel's epilogue).
    Asynchronous on ``stream`` (default: the current stream)."""
    a, b, c, d = (int(v) for v in pattern)
    lib = _lib.load()
    if x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D CUDA tensor")
    if not (x.is_contiguous() and values.is_contiguous()):
        raise ValueError("x and values must be contiguous")
    if values.dtype != x.dtype or values.device != x.device:
        raise ValueError("values must match x in dtype and device")
    dt = ks_dtype_of(x, tf32)
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, a * b * d), dtype=x.dtype, device=x.device)
    elif not out.is_contiguous() or out.dtype != x.dtype or out.device != x.device:
        raise ValueError("out must be contiguous with x's dtype and device")
    bias_ptr = _bias_ptr(bias, x, a * b * d)
    with torch.cuda.device(x.device):
        st = lib.ks_matmul_ep(x.data_ptr(), values.data_ptr(), a, b, c, d, batch, out.data_ptr(), dt, bias_ptr,
                              _act(act), _variant(variant), _stream_ptr(stream, x.device))
    _lib.check(st)
    return out


def matmul_host(x: torch.Tensor, values: torch.Tensor, pattern: Pattern, *, out: Optional[torch.Tensor] = None,
                tf32: bool = False, device: Optional[torch.device] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Y = X K^T for CPU tensors x (batch, a*c*d) and values, computed on the
    GPU (``device``, default the current one) with the rows streamed through in
    chunks whose copies overlap the products (pinned x, values and out give the
    overlap).  Asynchronous on ``stream``: synchronise it before reading out."""
    a, b, c, d = (int(v) for v in pattern)
    if x.dim() != 2 or x.is_cuda or values.is_cuda:
        raise ValueError("x must be a 2-D CPU tensor and values a CPU tensor")
    if not (x.is_contiguous() and values.is_contiguous()) or values.dtype != x.dtype:
        raise ValueError("x and values must be contiguous, with one dtype")
    dt = ks_dtype_of(x, tf32)
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, a * b * d), dtype=x.dtype, pin_memory=x.is_pinned())
    elif out.is_cuda or not out.is_contiguous() or out.dtype != x.dtype or out.shape != (batch, a * b * d):
        raise ValueError("out must be a contiguous CPU tensor (batch, a*b*d) with x's dtype")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        st = _lib.load().ks_matmul_host(x.data_ptr(), values.data_ptr(), a, b, c, d, batch, out.data_ptr(), dt,
                                        _stream_ptr(stream, dev))
    _lib.check(st)
    return out


def _act(act: str) -> int:
    if act not in _lib.ACTIVATIONS:
        raise ValueError(f"act must be one of {sorted(_lib.ACTIVATIONS)}")
    return _lib.ACTIVATIONS[act]


def _bias_ptr(bias: Optional[torch.Tensor], x: torch.Tensor, n: int):
    if bias is None:
        return None
    if bias.dtype != x.dtype or bias.device != x.device or not bias.is_contiguous() or bias.numel() != n:
        raise ValueError(f"bias must be a contiguous tensor of {n} elements with x's dtype and device")
    return bias.data_ptr()


def _check_pair(u: torch.Tensor, v: torch.Tensor, names: str) -> None:
    if u.dim() != 2 or not u.is_cuda or not u.is_contiguous() or not v.is_contiguous():
        raise ValueError(f"{names} must be contiguous CUDA tensors, the first 2-D")
    if v.dtype != u.dtype or v.device != u.device:
        raise ValueError(f"{names} must share dtype and device")


def matmul_dx(dy: torch.Tensor, values: torch.Tensor, pattern: Pattern, *, out: Optional[torch.Tensor] = None,
              tf32: bool = False, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Input gradient of Y = X K^T: dX = dY K, (batch, a*c*d) from dY (batch, a*b*d)."""
    a, b, c, d = (int(v) for v in pattern)
    _check_pair(dy, values, "dy and values")
    if out is None:
        out = torch.empty((dy.shape[0], a * c * d), dtype=dy.dtype, device=dy.device)
    with torch.cuda.device(dy.device):
        st = _lib.load().ks_matmul_dx(dy.data_ptr(), values.data_ptr(), a, b, c, d, dy.shape[0], out.data_ptr(),
                                      ks_dtype_of(dy, tf32), _stream_ptr(stream, dy.device))
    _lib.check(st)
    return out


def matmul_dv(dy: torch.Tensor, x: torch.Tensor, pattern: Pattern, *, out: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Values gradient of Y = X K^T: dV[i][l][k][j] = sum_n dY[n,(i,k,l)] X[n,(i,j,l)],
    a tensor of shape (a, d, b, c) (fp32 sums; bf16 rounded once)."""
    a, b, c, d = (int(v) for v in pattern)
    _check_pair(dy, x, "dy and x")
    if x.shape[0] != dy.shape[0]:
        raise ValueError("dy and x need the same number of rows")
    if out is None:
        out = torch.empty((a, d, b, c), dtype=dy.dtype, device=dy.device)
    with torch.cuda.device(dy.device):
        st = _lib.load().ks_matmul_dv(dy.data_ptr(), x.data_ptr(), a, b, c, d, dy.shape[0], out.data_ptr(),
                                      ks_dtype_of(dy), _stream_ptr(stream, dy.device))
    _lib.check(st)
    return out


def bias_grad(dy: torch.Tensor, *, out: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Column sums of dY (batch, width): the bias gradient of y = x K^T + bias
    (fp32 sums in a fixed order; bf16 rounded once)."""
    if dy.dim() != 2 or not dy.is_cuda or not dy.is_contiguous():
        raise ValueError("dy must be a contiguous 2-D CUDA tensor")
    if out is None:
        out = torch.empty(dy.shape[1], dtype=dy.dtype, device=dy.device)
    elif out.numel() != dy.shape[1] or out.dtype != dy.dtype or out.device != dy.device or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor of width elements with dy's dtype and device")
    with torch.cuda.device(dy.device):
        st = _lib.load().ks_bias_grad(dy.data_ptr(), dy.shape[0], dy.shape[1], out.data_ptr(), ks_dtype_of(dy),
                                      _stream_ptr(stream, dy.device))
    _lib.check(st)
    return out


def butterfly_factorize(a: torch.Tensor, *, stream: Optional[torch.cuda.Stream] = None):
    """Fit a dense 2^L x 2^L fp32 CUDA matrix A (the K of Y = X K^T) with the L
    butterfly factors; returns (factors, patterns) for chain(), factor 0 first."""
    if a.dim() != 2 or a.shape[0] != a.shape[1] or not a.is_cuda or not a.is_contiguous():
        raise ValueError("a must be a square contiguous CUDA matrix")
    n = a.shape[0]
    L = n.bit_length() - 1
    if n != 1 << L or L < 1:
        raise ValueError("the size must be a power of two")
    patterns = [(2 ** (k - 1), 2, 2, 2 ** (L - k)) for k in range(1, L + 1)]
    factors = [torch.empty(p[0] * p[1] * p[2] * p[3], dtype=a.dtype, device=a.device) for p in patterns]
    ptrs = (ctypes.c_void_p * L)(*[f.data_ptr() for f in factors])
    with torch.cuda.device(a.device):
        st = _lib.load().ks_butterfly_factorize(a.data_ptr(), L, ptrs, ks_dtype_of(a), _stream_ptr(stream, a.device))
    _lib.check(st)
    return factors, patterns


class _KSLinearFn(torch.autograd.Function):
    """Y = X K^T with K the KS factor of `pattern`; both gradients on the GPU."""

    @staticmethod
    def forward(ctx, x, values, bias, pattern):
        ctx.pattern = pattern
        ctx.save_for_backward(x, values)
        return matmul(x, values.contiguous(), pattern, bias=bias)  # bias fused into the epilogue

    @staticmethod
    def backward(ctx, dy):
        x, values = ctx.saved_tensors
        dy = dy.contiguous()
        dx = matmul_dx(dy, values.contiguous(), ctx.pattern) if ctx.needs_input_grad[0] else None
        dv = matmul_dv(dy, x, ctx.pattern).view(values.shape) if ctx.needs_input_grad[1] else None
        db = bias_grad(dy) if ctx.needs_input_grad[2] else None
        return dx, dv, db, None


class KSLinear(torch.nn.Module):
    """A linear layer whose weight is one KS factor of pattern (a, b, c, d):
    in_features a*c*d, out_features a*b*d, y = x K^T (+ bias, fused into the
    product's epilogue; its gradient is the column sum of dY, ks_bias_grad).
    The values are a parameter of shape (a, d, b, c), drawn N(0, 1/c)
    (unit-variance outputs for unit-variance inputs).  Leading dimensions of x
    are flattened."""

    def __init__(self, pattern: Pattern, bias: bool = False, dtype=torch.float32, device=None):
        super().__init__()
        a, b, c, d = (int(v) for v in pattern)
        self.pattern = (a, b, c, d)
        self.in_features, self.out_features = a * c * d, a * b * d
        self.values = torch.nn.Parameter(torch.randn(a, d, b, c, dtype=dtype, device=device) * (1.0 / c) ** 0.5)
        self.bias = torch.nn.Parameter(torch.zeros(a * b * d, dtype=dtype, device=device)) if bias else None

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        y = _KSLinearFn.apply(x.reshape(-1, self.in_features).contiguous(), self.values, self.bias, self.pattern)
        return y.reshape(*lead, self.out_features)


def chain(x: torch.Tensor, factors: Sequence[torch.Tensor], patterns: Sequence[Pattern], *,
          out: Optional[torch.Tensor] = None, tf32: bool = False, fused: bool = True,
          bias: Optional[torch.Tensor] = None, act: str = "none",
          stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Y = act(X (K_{n-1} ... K_0)^T + bias), factor 0 applied first, the
    epilogue fused into the last factor's kernel.  fused=False forces one
    kernel per factor (KS_CHAIN_UNFUSED).  Two factors with bias and GELU are
    a Monarch-style MLP layer."""
    lib = _lib.load()
    n = len(factors)
    if n == 0 or len(patterns) != n:
        raise ValueError("need one pattern per factor")
    if x.dim() != 2 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D CUDA tensor")
    for f in factors:
        if f.dtype != x.dtype or f.device != x.device or not f.is_contiguous():
            raise ValueError("factors must be contiguous, with x's dtype and device")
    dt = ks_dtype_of(x, tf32)
    a, b, c, d = (int(v) for v in patterns[-1])
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, a * b * d), dtype=x.dtype, device=x.device)
    ptrs = (ctypes.c_void_p * n)(*[f.data_ptr() for f in factors])
    pats = (KsPattern * n)(*[KsPattern(*[int(v) for v in p]) for p in patterns])
    with torch.cuda.device(x.device):
        st = lib.ks_chain_ep(x.data_ptr(), ptrs, pats, n, batch, out.data_ptr(), dt, 0 if fused else KS_CHAIN_UNFUSED,
                             _bias_ptr(bias, x, a * b * d), _act(act), _stream_ptr(stream, x.device))
    _lib.check(st)
    return out


def plan(pattern: Pattern, batch: int, dtype: int = KS_F32) -> str:
    """Name of the kernel family the heuristic picks (host only)."""
    v = ctypes.c_int(-1)
    a, b, c, d = (int(t) for t in pattern)
    _lib.check(_lib.load().ks_plan(a, b, c, d, int(batch), int(dtype), ctypes.byref(v)))
    return {v_: k for k, v_ in VARIANTS.items()}[v.value]


def workspace_info() -> Tuple[int, int]:
    """(allocations, reserved_bytes): workspace allocations the library has made
    from its pools since the process started (all devices), and the device
    memory the current device's pool holds now."""
    n, r = ctypes.c_int64(0), ctypes.c_int64(0)
    _lib.check(_lib.load().ks_workspace_info(ctypes.byref(n), ctypes.byref(r)))
    return int(n.value), int(r.value)


def sync_status(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Synchronise and raise KsError if a kernel reported a device-side failure."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _lib.check(_lib.load().ks_sync_status(_stream_ptr(stream, dev)))
