"""CPU oracle for the KroQuant online activation quantizer (ctypes binding).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the package smoke
check (``__graft_entry__.smoke``) and the benchmark's CPU-baseline leg may
import this package.  The product path never routes through it.

Every function takes and returns numpy arrays; the arithmetic lives in
``kq_oracle.c`` (plain scalar C, double precision), whose header lists the
sources and the readings it follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        ci = ctypes.c_int
        L.oracle_abi_version.restype = ci
        L.oracle_num_threads.restype = ci
        L.oracle_set_threads.argtypes = [ci]
        L.oracle_kron_expand.argtypes = [p, p]
        L.oracle_inverse32.argtypes = [p, p]
        L.oracle_inverse32.restype = ci
        L.oracle_e8m0.argtypes = [ctypes.c_float]
        L.oracle_e8m0.restype = ctypes.c_uint8
        L.oracle_e2m1.argtypes = [ctypes.c_double]
        L.oracle_e2m1.restype = ctypes.c_uint8
        L.oracle_mx_block.argtypes = [p, p, p]
        L.oracle_kq_transform.argtypes = [p, p, ci, i64, i64, p, p]
        L.oracle_kq_transform.restype = ci
        L.oracle_kq_quantize.argtypes = [p, p, ci, i64, i64, p, p]
        L.oracle_kq_quantize.restype = ci
        L.oracle_sq_quantize.argtypes = [p, p, i64, i64, p, p]
        L.oracle_sq_quantize.restype = ci
        L.oracle_mx_quantize.argtypes = [p, i64, i64, p, p]
        L.oracle_mx_quantize.restype = ci
        L.oracle_fold_weights.argtypes = [p, p, ci, p, p, i64, i64]
        L.oracle_fold_weights.restype = ci
        L.oracle_lu_factor.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_double, p]
        L.oracle_kron_expand_lu.argtypes = [p, p]
        L.oracle_kq_transform_lu.argtypes = [p, p, ci, i64, i64, p, p]
        L.oracle_kq_transform_lu.restype = ci
        L.oracle_kq_quantize_lu.argtypes = [p, p, ci, i64, i64, p, p]
        L.oracle_kq_quantize_lu.restype = ci
        L.oracle_fwht_transform.argtypes = [p, i64, i64, i64, p, p, p, p]
        L.oracle_fwht_transform.restype = ci
        L.oracle_mx_dequantize.argtypes = [p, p, i64, i64, p]
        L.oracle_mx_dequantize.restype = ci
        L.oracle_kq_inverse.argtypes = [p, p, ci, i64, i64, p, p]
        L.oracle_kq_inverse.restype = ci
        L.oracle_norm_kq.argtypes = [p, p, p, i64, ctypes.c_double, p, ci, i64, i64, p, p, p, p]
        L.oracle_norm_kq.restype = ci
        L.oracle_sf_offset.argtypes = [i64, i64, i64]
        L.oracle_sf_offset.restype = i64
        L.oracle_sf_bytes.argtypes = [i64, i64]
        L.oracle_sf_bytes.restype = i64
        L.oracle_scales_to_sf.argtypes = [p, i64, i64, p]
        L.oracle_scales_to_sf.restype = ci
        L.oracle_mx_quantize_f32.argtypes = [p, i64, i64, p, p]
        L.oracle_mx_quantize_f32.restype = ci
        L.oracle_mxf4_gemm.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, p]
        L.oracle_mxf4_gemm.restype = ci
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def kron_expand(F):
    """Dense 32x32 K = G1 (x) ... (x) G5 (float64) from a [5,2,2] float32 factor set."""
    F = _c(F, np.float32).reshape(5, 2, 2)
    K = np.empty((32, 32), np.float64)
    lib().oracle_kron_expand(_ptr(F), _ptr(K))
    return K


def inverse32(A):
    A = _c(A, np.float64).reshape(32, 32)
    out = np.empty((32, 32), np.float64)
    if lib().oracle_inverse32(_ptr(A), _ptr(out)) != 0:
        raise ValueError("singular 32x32 matrix")
    return out


def e8m0(amax: float) -> int:
    return int(lib().oracle_e8m0(float(amax)))


def e2m1(v: float) -> int:
    return int(lib().oracle_e2m1(float(v)))


def mx_block(y):
    y = _c(y, np.float32).reshape(32)
    codes = np.empty(16, np.uint8)
    scale = np.empty(1, np.uint8)
    lib().oracle_mx_block(_ptr(y), _ptr(codes), _ptr(scale))
    return codes, int(scale[0])


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with status {rc}")


def _shape(x):
    if x.ndim != 2:
        raise ValueError("activation must be 2-D [M, d]")
    return x.shape


def kq_transform(x_bf16, factors, shared=False, want_absbound=False):
    """fp32 y = T x per block (dense, double, rounded once), optionally with |K||x|."""
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    f = _c(factors, np.float32)
    y = np.empty((M, d), np.float32)
    ab = np.empty((M, d), np.float64) if want_absbound else None
    _check(lib().oracle_kq_transform(_ptr(x), _ptr(f), int(bool(shared)), M, d, _ptr(y), _ptr(ab)),
           "kq_transform")
    return (y, ab) if want_absbound else y


def kq_quantize(x_bf16, factors, shared=False):
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    f = _c(factors, np.float32)
    codes = np.empty((M, d // 2), np.uint8)
    scales = np.empty((M, d // 32), np.uint8)
    _check(lib().oracle_kq_quantize(_ptr(x), _ptr(f), int(bool(shared)), M, d, _ptr(codes), _ptr(scales)),
           "kq_quantize")
    return codes, scales


def sq_quantize(x_bf16, mult):
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    m = _c(mult, np.float32)
    codes = np.empty((M, d // 2), np.uint8)
    scales = np.empty((M, d // 32), np.uint8)
    _check(lib().oracle_sq_quantize(_ptr(x), _ptr(m), M, d, _ptr(codes), _ptr(scales)), "sq_quantize")
    return codes, scales


def mx_quantize(x_bf16):
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    codes = np.empty((M, d // 2), np.uint8)
    scales = np.empty((M, d // 32), np.uint8)
    _check(lib().oracle_mx_quantize(_ptr(x), M, d, _ptr(codes), _ptr(scales)), "mx_quantize")
    return codes, scales


def fold_weights(W, factors, shared=False, want_absbound=False):
    """W' = W T^-1 (fp32 result of a double computation), optionally with |W||K^-1|."""
    W = _c(W, np.float32)
    N, d = _shape(W)
    f = _c(factors, np.float32)
    out = np.empty((N, d), np.float32)
    ab = np.empty((N, d), np.float64) if want_absbound else None
    _check(lib().oracle_fold_weights(_ptr(W), _ptr(f), int(bool(shared)), _ptr(out), _ptr(ab), N, d),
           "fold_weights")
    return (out, ab) if want_absbound else out


def lu_factor(a, b, c):
    """G = L U of one factor (double) from its LU scalars."""
    G = np.empty((2, 2), np.float64)
    lib().oracle_lu_factor(float(a), float(b), float(c), _ptr(G))
    return G


def kron_expand_lu(params):
    """Dense 32x32 K (float64) from [5, 3] float32 LU scalars (a, b, c) per factor."""
    P = _c(params, np.float32).reshape(5, 3)
    K = np.empty((32, 32), np.float64)
    lib().oracle_kron_expand_lu(_ptr(P), _ptr(K))
    return K


def kq_transform_lu(x_bf16, params, shared=False, want_absbound=False):
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    P = _c(params, np.float32)
    y = np.empty((M, d), np.float32)
    ab = np.empty((M, d), np.float64) if want_absbound else None
    _check(lib().oracle_kq_transform_lu(_ptr(x), _ptr(P), int(bool(shared)), M, d, _ptr(y), _ptr(ab)),
           "kq_transform_lu")
    return (y, ab) if want_absbound else y


def kq_quantize_lu(x_bf16, params, shared=False):
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    P = _c(params, np.float32)
    codes = np.empty((M, d // 2), np.uint8)
    scales = np.empty((M, d // 32), np.uint8)
    _check(lib().oracle_kq_quantize_lu(_ptr(x), _ptr(P), int(bool(shared)), M, d, _ptr(codes), _ptr(scales)),
           "kq_quantize_lu")
    return codes, scales


def fwht_transform(x_bf16, H, want_absbound=False):
    """fp32 y = H_H x / sqrt(H) per H-block (double, rounded once), optionally with the error scale."""
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    y = np.empty((M, d), np.float32)
    ab = np.empty((M, d), np.float64) if want_absbound else None
    _check(lib().oracle_fwht_transform(_ptr(x), int(H), M, d, _ptr(y), _ptr(ab), None, None), "fwht_transform")
    return (y, ab) if want_absbound else y


def fwht_quantize(x_bf16, H):
    x = _c(x_bf16, np.uint16)
    M, d = _shape(x)
    codes = np.empty((M, d // 2), np.uint8)
    scales = np.empty((M, d // 32), np.uint8)
    _check(lib().oracle_fwht_transform(_ptr(x), int(H), M, d, None, None, _ptr(codes), _ptr(scales)),
           "fwht_quantize")
    return codes, scales


def mx_dequantize(codes, scales):
    """fp32 [M, d] decode of MXFP4 codes [M, d/2] and E8M0 scales [M, d/32]."""
    c = _c(codes, np.uint8)
    sc = _c(scales, np.uint8)
    M, d = c.shape[0], c.shape[1] * 2
    out = np.empty((M, d), np.float32)
    _check(lib().oracle_mx_dequantize(_ptr(c), _ptr(sc), M, d, _ptr(out)), "mx_dequantize")
    return out


def kq_inverse(y, factors, shared=False, want_absbound=False):
    """x = K^-1 y per 32-block (double Gauss-Jordan inverse, rounded once to fp32)."""
    yv = _c(y, np.float32)
    M, d = _shape(yv)
    f = _c(factors, np.float32)
    x = np.empty((M, d), np.float32)
    ab = np.empty((M, d), np.float64) if want_absbound else None
    _check(lib().oracle_kq_inverse(_ptr(yv), _ptr(f), int(bool(shared)), M, d, _ptr(x), _ptr(ab)), "kq_inverse")
    return (x, ab) if want_absbound else x


def norm_kq(h_bf16, gamma, beta, eps, factors, shared=False, want=("codes",)):
    """LayerNorm + AdaLN modulation + KroQuant quantizer (double), see kq_oracle.c R9.

    gamma, beta: [nsamples, d] float32.  `want` picks outputs among
    "codes" (codes, scales), "y" (fp32 transform) and "absb" (|K||x_mod|).
    """
    h = _c(h_bf16, np.uint16)
    M, d = _shape(h)
    g = _c(gamma, np.float32)
    b = _c(beta, np.float32)
    ns = g.shape[0]
    f = _c(factors, np.float32)
    y = np.empty((M, d), np.float32) if "y" in want else None
    ab = np.empty((M, d), np.float64) if "absb" in want else None
    codes = np.empty((M, d // 2), np.uint8) if "codes" in want else None
    scales = np.empty((M, d // 32), np.uint8) if "codes" in want else None
    _check(lib().oracle_norm_kq(_ptr(h), _ptr(g), _ptr(b), ns, float(eps), _ptr(f), int(bool(shared)), M, d,
                                _ptr(y), _ptr(ab), _ptr(codes), _ptr(scales)), "norm_kq")
    out = {}
    if codes is not None:
        out["codes"], out["scales"] = codes, scales
    if y is not None:
        out["y"] = y
    if ab is not None:
        out["absb"] = ab
    return out


def sf_offset(r: int, j: int, nb: int) -> int:
    """Byte offset of the scale (row r, block column j) in the scale-factor layout."""
    return int(lib().oracle_sf_offset(r, j, nb))


def sf_bytes(rows: int, nb: int) -> int:
    """Size of a scale-factor-layout buffer for rows x nb scales (whole 512-byte units)."""
    return int(lib().oracle_sf_bytes(rows, nb))


def scales_to_sf(scales, fill=None):
    """Row-major scales [rows, nb] -> scale-factor layout (uint8, sf_bytes long).

    Entries the layout leaves undefined hold `fill` (default: 0xFF, so a test
    that reads them by mistake sees NaN scales); the pad of an odd nb is 0x00.
    """
    sc = _c(scales, np.uint8)
    rows, nb = sc.shape
    out = np.full(sf_bytes(rows, nb), 0xFF if fill is None else fill, np.uint8)
    _check(lib().oracle_scales_to_sf(_ptr(sc), rows, nb, _ptr(out)), "scales_to_sf")
    return out


def sf_defined_mask(rows: int, nb: int):
    """Boolean mask over an SF buffer: the bytes scales_to_sf defines."""
    mask = np.zeros(sf_bytes(rows, nb), bool)
    r = np.arange(rows)[:, None]
    cols = nb + 1 if nb % 2 else nb
    j = np.arange(cols)[None, :]
    ka = (nb + 3) // 4
    off = ((r // 128) * ka + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)
    mask[off.ravel()] = True
    return mask


def mx_quantize_f32(x):
    """Plain MXFP4 quantizer on fp32 input: (codes [M, d/2], scales [M, d/32])."""
    xv = _c(x, np.float32)
    M, d = _shape(xv)
    codes = np.empty((M, d // 2), np.uint8)
    scales = np.empty((M, d // 32), np.uint8)
    _check(lib().oracle_mx_quantize_f32(_ptr(xv), M, d, _ptr(codes), _ptr(scales)), "mx_quantize_f32")
    return codes, scales


def mxf4_gemm(codes_a, scales_a, codes_b, scales_b, rows=None, want_absbound=False):
    """D = A B^T over decoded MXFP4 operands, in double (kq_oracle.c R10).

    codes_a [M, K/2], scales_a [M, K/32] (row-major), likewise B [N, ...].
    `rows` restricts the output to those rows of A (sampled checks).
    """
    ca, sa = _c(codes_a, np.uint8), _c(scales_a, np.uint8)
    cb, sb = _c(codes_b, np.uint8), _c(scales_b, np.uint8)
    M, K = ca.shape[0], ca.shape[1] * 2
    N = cb.shape[0]
    assert cb.shape[1] * 2 == K and sa.shape == (M, K // 32) and sb.shape == (N, K // 32)
    ms = None if rows is None else _c(rows, np.int64)
    nm = M if ms is None else ms.size
    D = np.empty((nm, N), np.float64)
    ab = np.empty((nm, N), np.float64) if want_absbound else None
    _check(lib().oracle_mxf4_gemm(_ptr(ca), _ptr(sa), _ptr(cb), _ptr(sb), _ptr(ms), nm, M, N, K, _ptr(D), _ptr(ab)),
           "mxf4_gemm")
    return (D, ab) if want_absbound else D
