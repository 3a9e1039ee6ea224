"""The C-ABI library loads, exports every declared entry point, and its host-side
argument checks return the documented status before touching CUDA (no GPU).

Every call below is built to FAIL validation (or to be an M == 0 no-op): none
may pass its checks with the placeholder pointers used here, because a call
that passes would launch a kernel on them.
"""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def L():
    from w4a4_mxfp4_post_b200 import build

    build.build()
    import w4a4_mxfp4_post_b200 as kq

    return kq.lib()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(HEADER_DIR, fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M):
            if m.group(1) not in ("if", "return", "sizeof"):
                names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kq_quantize", "kq_quantize_shared", "sq_quantize", "mx_quantize", "kq_fold_weights",
                     "kq_transform_f32", "kq_quantize_variant", "kq_last_error", "kq_abi_version"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    from w4a4_mxfp4_post_b200 import LIB_PATH

    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert getattr(L, n) is not None


def test_python_binding_mirrors_every_declared_entry_point():
    """The binding is thin and complete: one Python function per C entry point, same name."""
    import w4a4_mxfp4_post_b200 as kq

    missing = [n for n in declared_functions() if not callable(getattr(kq, n, None))]
    assert not missing, missing
    assert set(declared_functions()) <= set(kq.__all__) | {"kq_last_error", "kq_abi_version"}


def test_abi_version(L):
    assert L.kq_abi_version() == 1


def err(L):
    return L.kq_last_error().decode()


P = ctypes.c_void_p


def test_shape_errors_before_cuda(L):
    assert L.kq_quantize(P(16), P(16), P(16), P(16), 4, 33, None) == -2
    assert "multiple of 32" in err(L)
    assert L.kq_quantize(P(16), P(16), P(16), P(16), -1, 64, None) == -2
    assert L.sq_quantize(P(16), P(16), P(16), P(16), 4, 0, None) == -2
    assert L.mx_quantize(P(16), P(16), P(16), 4, -32, None) == -2
    assert L.kq_fold_weights(P(16), P(16), 0, P(16), 4, 48, None) == -2
    assert L.kq_transform_f32(P(16), P(16), 0, P(16), 4, 31, None) == -2
    # overflow of M * d
    assert L.mx_quantize(P(16), P(16), P(16), 2 ** 62, 64, None) == -2


def test_empty_is_a_noop(L):
    for M in (0,):
        assert L.kq_quantize(None, None, None, None, M, 64, None) == 0
        assert L.kq_quantize_shared(None, None, None, None, M, 64, None) == 0
        assert L.sq_quantize(None, None, None, None, M, 64, None) == 0
        assert L.mx_quantize(None, None, None, M, 64, None) == 0
        assert L.kq_fold_weights(None, None, 0, None, M, 64, None) == 0
        assert L.kq_transform_f32(None, None, 0, None, M, 64, None) == 0
        assert err(L) == ""


def test_null_errors(L):
    assert L.kq_quantize(None, P(16), P(16), P(16), 4, 64, None) == -1
    assert L.kq_quantize(P(16), None, P(16), P(16), 4, 64, None) == -1
    assert L.kq_quantize(P(16), P(16), None, P(16), 4, 64, None) == -1
    assert L.kq_quantize(P(16), P(16), P(16), None, 4, 64, None) == -1
    assert L.sq_quantize(P(16), None, P(16), P(16), 4, 64, None) == -1
    assert L.mx_quantize(P(16), P(16), None, 4, 64, None) == -1
    assert L.kq_fold_weights(P(16), P(16), 0, None, 4, 64, None) == -1
    assert L.kq_transform_f32(P(16), P(16), 0, None, 4, 64, None) == -1
    assert "NULL" in err(L)


def test_alignment_errors(L):
    assert L.kq_quantize(P(8), P(16), P(16), P(16), 4, 64, None) == -3
    assert L.kq_quantize(P(16), P(4), P(16), P(16), 4, 64, None) == -3
    assert L.kq_quantize(P(16), P(16), P(24), P(16), 4, 64, None) == -3
    assert L.sq_quantize(P(16), P(20), P(16), P(16), 4, 64, None) == -3
    assert L.kq_fold_weights(P(16), P(16), 0, P(40), 4, 64, None) == -3
    assert "aligned" in err(L)


def test_variant_errors_before_cuda(L):
    assert L.kq_quantize_variant(10, P(16), P(16), 0, P(16), P(16), 4, 64, None) == -5
    for retired in (5, 6, 7, 8):
        assert L.kq_quantize_variant(retired, P(16), P(16), 0, P(16), P(16), 4, 64, None) == -5
    assert L.sq_quantize_variant(5, P(16), P(16), P(16), P(16), 4, 64, None) == -5
    assert L.mx_quantize_variant(-1, P(16), P(16), P(16), 4, 64, None) == -5
    assert "variant" in err(L)
    assert L.kq_wait_timeouts(None, 0) == -1


def test_lu_and_fwht_argument_errors(L):
    assert L.kq_quantize_lu(P(16), None, 0, P(16), P(16), 4, 64, None) == -1
    assert L.kq_quantize_lu(P(16), P(16), 0, P(16), P(16), 4, 40, None) == -2
    assert L.kq_quantize_lu(P(16), P(2), 0, P(16), P(16), 4, 64, None) == -3
    assert L.fwht_quantize(P(16), 48, P(16), P(16), 4, 96, None) == -2
    assert L.fwht_quantize(P(16), 64, P(16), P(16), 4, 96, None) == -2
    assert L.fwht_quantize(P(16), 2048, P(16), P(16), 4, 2048, None) == -2
    assert L.fwht_quantize(P(16), 32, None, P(16), 4, 64, None) == -1
    assert L.kq_quantize_lu(None, None, 0, None, None, 0, 64, None) == 0
    assert L.fwht_quantize(None, 32, None, None, 0, 64, None) == 0


def test_norm_inverse_dequant_argument_errors(L):
    import ctypes as C

    f = C.c_float
    assert L.norm_kq_quantize(P(16), P(16), P(16), 2, f(1e-6), P(16), 0, P(16), P(16), 5, 64, None) == -2
    assert L.norm_kq_quantize(P(16), P(16), P(16), 1, f(1e-6), P(16), 0, P(16), P(16), 4, 32 * 513, None) == -2
    assert L.norm_kq_quantize(P(16), None, P(16), 1, f(1e-6), P(16), 0, P(16), P(16), 4, 64, None) == -1
    assert L.norm_kq_quantize(P(16), P(8), P(16), 1, f(1e-6), P(16), 0, P(16), P(16), 4, 64, None) == -3
    assert L.norm_kq_quantize(P(16), P(16), P(16), 1, f(-1.0), P(16), 0, P(16), P(16), 4, 64, None) == -2
    # the variant export: same checks, then the variant number
    assert L.norm_kq_quantize_variant(1, P(16), P(16), P(16), 2, f(1e-6), P(16), 0, P(16), P(16), 5, 64, None) == -2
    assert L.norm_kq_quantize_variant(9, P(16), P(16), P(16), 1, f(1e-6), P(16), 0, P(16), P(16), 4, 64, None) == -5
    assert L.kq_inverse_f32(P(16), P(16), 0, None, 4, 64, None) == -1
    assert L.kq_inverse_f32(P(16), P(16), 0, P(16), 4, 40, None) == -2
    assert L.mx_dequantize(P(16), P(16), P(8), 4, 64, None) == -3
    assert L.mx_dequantize(None, None, None, 0, 64, None) == 0


def test_w4a4_argument_errors(L):
    L.kq_sf_bytes.restype = ctypes.c_int64
    L.kq_sf_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
    assert L.kq_sf_bytes(300, 2240) == 3 * 18 * 512
    assert L.kq_sf_bytes(0, 64) == 0
    assert L.kq_sf_bytes(4, 40) == -1
    # kq_quantize_sf
    assert L.kq_quantize_sf(P(16), P(16), 0, P(16), P(16), 4, 40, None) == -2
    assert L.kq_quantize_sf(P(16), None, 0, P(16), P(16), 4, 64, None) == -1
    assert L.kq_quantize_sf(P(8), P(16), 0, P(16), P(16), 4, 64, None) == -3
    assert L.kq_quantize_sf(None, None, 0, None, None, 0, 64, None) == 0
    # mx_quantize_f32
    assert L.mx_quantize_f32(P(16), P(16), P(16), 2, 4, 64, None) == -2
    assert L.mx_quantize_f32(P(16), P(16), P(16), 0, 4, 48, None) == -2
    assert L.mx_quantize_f32(P(16), None, P(16), 1, 4, 64, None) == -1
    assert L.mx_quantize_f32(P(16), P(8), P(16), 1, 4, 64, None) == -3
    assert L.mx_quantize_f32(None, None, None, 1, 0, 64, None) == 0
    # mx_scales_to_sf
    assert L.mx_scales_to_sf(P(16), P(16), -1, 64, None) == -2
    assert L.mx_scales_to_sf(None, P(16), 4, 64, None) == -1
    assert L.mx_scales_to_sf(None, None, 0, 64, None) == 0
    # mxf4_gemm: a_codes, a_sf, b_codes, b_sf, out, out_f32, M, N, K, stream
    assert L.mxf4_gemm(P(16), P(16), P(16), P(16), P(16), 0, 4, 8, 48, None) == -2      # K % 32
    assert L.mxf4_gemm(P(16), P(16), P(16), P(16), P(16), 0, 4, 12, 64, None) == -2     # N % 8
    assert L.mxf4_gemm(P(16), P(16), P(16), P(16), P(16), 0, 4, 8, 0, None) == -2       # K <= 0
    assert L.mxf4_gemm(P(16), P(16), P(16), P(16), P(16), 0, 1 << 31, 8, 64, None) == -2
    assert L.mxf4_gemm(P(16), None, P(16), P(16), P(16), 0, 4, 8, 64, None) == -1
    assert L.mxf4_gemm(P(16), P(16), P(16), P(8), P(16), 0, 4, 8, 64, None) == -3
    assert L.mxf4_gemm(P(16), P(16), P(16), P(16), P(4), 1, 4, 8, 64, None) == -3
    assert L.mxf4_gemm(None, None, None, None, None, 0, 0, 8, 64, None) == 0
    assert L.mxf4_gemm(None, None, None, None, None, 0, 4, 0, 64, None) == 0
    # tile configurations 0-8 exist; others are a variant error (checked before any launch)
    assert L.mxf4_gemm_variant(9, P(16), P(16), P(16), P(16), P(16), 0, 4, 8, 64, None) == -5
    assert L.mxf4_gemm_variant(-1, P(16), P(16), P(16), P(16), P(16), 0, 4, 8, 64, None) == -5
    # norm_kq_quantize_sf: h, gamma, beta, nsamples, eps, factors, shared, codes, sf, M, d, stream
    f = ctypes.c_float
    assert L.norm_kq_quantize_sf(P(16), P(16), P(16), 2, f(1e-6), P(16), 0, P(16), P(16), 5, 64, None) == -2
    assert L.norm_kq_quantize_sf(P(16), P(16), P(16), 1, f(1e-6), P(16), 0, P(16), None, 4, 64, None) == -1
    assert L.norm_kq_quantize_sf(P(16), P(8), P(16), 1, f(1e-6), P(16), 0, P(16), P(16), 4, 64, None) == -3
    assert L.norm_kq_quantize_sf(None, None, None, 1, f(1e-6), None, 0, None, None, 0, 64, None) == 0


def test_python_binding_rejects_cpu_tensors():
    import torch

    import w4a4_mxfp4_post_b200 as kq

    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kq.mx_quantize(x)
    with pytest.raises(TypeError):
        kq.mx_quantize(torch.zeros(4, 64))
