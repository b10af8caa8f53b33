"""The C ABI without a GPU: the library loads, exports every entry point that
include/ks.h declares, validates arguments on the host and plans kernels.
No call here reaches a CUDA API (all of them fail validation first)."""
import ctypes
import os
import re

import pytest

from kronecker_sparse_matrix_b200 import _lib, build as ksbuild
from kronecker_sparse_matrix_b200 import plan
from kronecker_sparse_matrix_b200.inputs import sweep_patterns, butterfly_patterns

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ks.h")


@pytest.fixture(scope="module")
def lib():
    ksbuild.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(ks_[a-z_]+)\s*\(", src, flags=re.M)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for n in ["ks_matmul", "ks_matmul_variant", "ks_chain", "ks_plan", "ks_last_error",
              "ks_status_string", "ks_sync_status", "ks_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding misses {name}"


def test_version_and_status_strings(lib):
    assert lib.ks_version() >= 100
    assert lib.ks_status_string(0) == b"KS_OK"
    assert lib.ks_status_string(6) == b"KS_ERR_TIMEOUT"
    assert lib.ks_status_string(99) == b"KS_ERR_UNKNOWN"


P = 1 << 20  # a fake 256-byte-aligned address; never dereferenced (validation fails first)


@pytest.mark.parametrize("pat", [(0, 1, 1, 1), (1, -2, 1, 1), (1, 1, 0, 1), (1, 1, 1, -1)])
def test_bad_pattern_is_invalid(lib, pat):
    assert lib.ks_matmul(P, P, *pat, 4, P * 8, 0, None) == 1
    assert b"positive" in lib.ks_last_error()


def test_negative_batch_bad_dtype_null_pointers(lib):
    assert lib.ks_matmul(P, P, 2, 2, 2, 2, -1, P * 8, 0, None) == 1
    assert lib.ks_matmul(P, P, 2, 2, 2, 2, 4, P * 8, 7, None) == 1
    assert lib.ks_matmul(None, P, 2, 2, 2, 2, 4, P * 8, 0, None) == 1
    assert lib.ks_matmul(P, P, 2, 2, 2, 2, 4, None, 0, None) == 1
    assert lib.ks_matmul_variant(P, P, 2, 2, 2, 2, 4, P * 8, 0, 9, None) == 1


def test_overflow_is_invalid(lib):
    big = 1 << 40
    assert lib.ks_matmul(P, P, big, big, 2, 2, 4, P * 8, 0, None) == 1
    assert b"overflow" in lib.ks_last_error() or b"2^31" in lib.ks_last_error()


def test_zero_batch_is_a_noop(lib):
    assert lib.ks_matmul(None, None, 2, 2, 2, 2, 0, None, 0, None) == 0


def test_misaligned_pointers(lib):
    assert lib.ks_matmul(P + 2, P, 2, 2, 2, 2, 4, P * 8, 0, None) == 2   # fp32 needs 4 bytes
    assert lib.ks_matmul(P, P, 2, 2, 2, 2, 4, P * 8 + 1, 2, None) == 2   # bf16 needs 2 bytes


def test_overlapping_output_is_invalid(lib):
    # Y = X: 4 rows of 8 fp32
    assert lib.ks_matmul(P, P * 4, 2, 2, 2, 2, 4, P, 0, None) == 1
    assert b"overlaps X" in lib.ks_last_error()
    assert lib.ks_matmul(P, P * 4, 2, 2, 2, 2, 4, P * 4 + 16, 0, None) == 1
    assert b"overlaps values" in lib.ks_last_error()


def test_chain_validation(lib):
    pats = (_lib.KsPattern * 2)(_lib.KsPattern(1, 2, 2, 2), _lib.KsPattern(1, 2, 2, 1))
    ptrs = (ctypes.c_void_p * 2)(P, P)
    assert lib.ks_chain(P, ptrs, pats, 2, 4, P * 8, 0, None) == 1
    assert b"input width" in lib.ks_last_error()
    assert lib.ks_chain(P, ptrs, pats, 0, 4, P * 8, 0, None) == 1
    ok = (_lib.KsPattern * 2)(_lib.KsPattern(1, 2, 2, 2), _lib.KsPattern(2, 2, 2, 1))
    null = (ctypes.c_void_p * 2)(P, None)
    assert lib.ks_chain(P, null, ok, 2, 4, P * 8, 0, None) == 1
    assert lib.ks_chain(P, ptrs, ok, 2, 0, P * 8, 0, None) == 0  # batch 0: no-op


def test_noalloc_chain_validates_on_the_host(lib):
    # the fixed scratch holds 16 MiB per intermediate: a 4096-wide fp32 intermediate fits
    # 1024 rows, and 1025 are refused before any device call
    pats = (_lib.KsPattern * 2)(_lib.KsPattern(1, 4096, 4096, 1), _lib.KsPattern(1, 4096, 4096, 1))
    ptrs = (ctypes.c_void_p * 2)(P, P)
    assert lib.ks_chain_noalloc(P, ptrs, pats, 2, 1025, P * 8, 0, None) == 1
    assert b"exceeds the fixed scratch" in lib.ks_last_error()
    bad = (_lib.KsPattern * 2)(_lib.KsPattern(1, 2, 2, 2), _lib.KsPattern(1, 2, 2, 1))
    assert lib.ks_chain_noalloc(P, ptrs, bad, 2, 4, P * 8, 0, None) == 1
    assert b"input width" in lib.ks_last_error()
    assert lib.ks_chain_noalloc(P, ptrs, pats, 2, 4, P * 8, 7, None) == 1  # unknown dtype
    assert lib.ks_chain_noalloc(P, (ctypes.c_void_p * 2)(P, None), pats, 2, 4, P * 8, 0, None) == 1
    assert lib.ks_chain_noalloc(P, ptrs, pats, 2, 0, P * 8, 0, None) == 0  # batch 0: no-op


def test_plan_is_host_only_and_sensible(lib):
    v = ctypes.c_int(-1)
    assert lib.ks_plan(1, 192, 48, 8, 25216, 0, ctypes.byref(v)) == 0
    assert v.value == _lib.KS_VARIANT_FMA
    for p in butterfly_patterns(12):
        assert plan(p, 4096) == "stream"
    for p in sweep_patterns():
        assert plan(p, 25088) == "fma"
    assert plan((3, 5, 7, 3), 10) == "stream"  # odd d: the scalar catch-all


def test_plan_sends_tf32_and_bf16_to_the_tensor_cores(lib):
    for p, n in [((1, 192, 48, 8), 25216), ((1, 256, 64, 16), 8192)]:
        assert plan(p, n, _lib.KS_TF32) == "tc"
        assert plan(p, n, _lib.KS_BF16) == "tc"
        assert plan(p, n, _lib.KS_F32) == "fma"  # fp32 keeps fp32 arithmetic
    for p in sweep_patterns():
        assert plan(p, 25088, _lib.KS_TF32) == "tc"
        assert plan(p, 25088, _lib.KS_BF16) == "tc"
    # TF32's K step is 8 j, bf16's 16
    assert plan((1, 64, 8, 1), 1000, _lib.KS_TF32) == "tc"
    assert plan((1, 64, 8, 1), 1000, _lib.KS_BF16) == "fma"
    assert plan((1, 64, 12, 1), 1000, _lib.KS_TF32) == "fma"
    assert plan((1, 64, 64, 3), 1000, _lib.KS_TF32) != "tc"  # d = 3: no l width for the tensor-core tiles
    for p in butterfly_patterns(12):
        assert plan(p, 4096, _lib.KS_TF32) == "stream"


def test_tc_variant_refuses_fp32(lib):
    v = ctypes.c_int(-1)
    assert lib.ks_plan(1, 64, 64, 1, 100, _lib.KS_F32, ctypes.byref(v)) == 0 and v.value == _lib.KS_VARIANT_FMA
    # forcing the tensor cores on KS_F32 is refused before any device call
    assert lib.ks_matmul_variant(P, P * 2, 1, 64, 64, 1, 100, P * 4, _lib.KS_F32, _lib.KS_VARIANT_TC, None) == 3
    assert b"KS_TF32" in lib.ks_last_error()


def test_injected_allocation_failure_is_reported_before_any_launch(lib, monkeypatch):
    n0 = ctypes.c_int64(-1)
    assert lib.ks_workspace_info(ctypes.byref(n0), None) == 0
    monkeypatch.setenv("KS_FAULT_INJECT", "alloc")
    pats = (_lib.KsPattern * 2)(_lib.KsPattern(1, 4, 4, 2), _lib.KsPattern(2, 4, 4, 1))
    ptrs = (ctypes.c_void_p * 2)(P * 2, P * 3)
    assert lib.ks_chain(P, ptrs, pats, 2, 4, P * 4, 0, None) == 4
    assert b"workspace" in lib.ks_last_error()
    assert lib.ks_matmul_dx(P, P * 2, 2, 2, 2, 2, 4, P * 4, 0, None) == 4
    assert lib.ks_matmul_dv(P, P * 2, 2, 2, 2, 2, 4, P * 4, 0, None) == 4
    facs = (ctypes.c_void_p * 4)(P * 4, P * 5, P * 6, P * 7)
    assert lib.ks_butterfly_factorize(P, 4, facs, 0, None) == 4
    n = ctypes.c_int64(-1)
    assert lib.ks_workspace_info(ctypes.byref(n), None) == 0 and n.value == n0.value  # nothing was allocated


def test_host_product_validates_on_the_host(lib):
    assert lib.ks_matmul_host(None, P, 2, 2, 2, 2, 4, P * 8, 0, None) == 1
    assert lib.ks_matmul_host(P, P, 2, 2, 2, 2, 4, P, 0, None) == 1  # Y overlaps X
    assert b"overlaps X" in lib.ks_last_error()
    assert lib.ks_matmul_host(P + 2, P * 4, 2, 2, 2, 2, 4, P * 8, 0, None) == 2
    assert lib.ks_matmul_host(None, None, 2, 2, 2, 2, 0, None, 0, None) == 0  # batch 0: no-op


def test_bias_grad_validates_on_the_host(lib):
    # dY at P (4 x 8 fp32 = 128 bytes), db elsewhere
    assert lib.ks_bias_grad(P, 4, 8, None, 0, None) == 1            # null db
    assert lib.ks_bias_grad(None, 4, 8, P * 8, 0, None) == 1        # null dY with rows to sum
    assert lib.ks_bias_grad(P, -1, 8, P * 8, 0, None) == 1          # negative batch
    assert lib.ks_bias_grad(P, 4, 0, P * 8, 0, None) == 1           # empty width
    assert lib.ks_bias_grad(P, 4, 8, P * 8, 7, None) == 1           # unknown dtype
    assert lib.ks_bias_grad(P, 1 << 62, 1 << 3, P * 8, 0, None) == 1  # sizes overflow
    assert lib.ks_bias_grad(P, 4, 8, P + 64, 0, None) == 1          # db inside dY
    assert b"overlaps" in lib.ks_last_error()
    assert lib.ks_bias_grad(P, 4, 8, P * 8 + 2, 0, None) == 2       # fp32 db not 4-byte aligned
    assert lib.ks_bias_grad(P + 1, 4, 8, P * 8, 2, None) == 2       # bf16 dY not 2-byte aligned


def test_fma_rate_probe_validates_on_the_host(lib):
    assert lib.ks_fma_rate_probe(None, 4, 16, None) == 1
    assert lib.ks_fma_rate_probe(P, 0, 16, None) == 1
    assert lib.ks_fma_rate_probe(P, 4, 24, None) == 1  # not a multiple of 16
    assert b"multiple of 16" in lib.ks_last_error()
    assert lib.ks_fma_rate_probe(P + 2, 4, 16, None) == 2


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load()
