"""KroQuant online activation quantizer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``include/kroquant.h`` (the shared
library ``libkroquant.so`` built in-tree by ``w4a4_mxfp4_post_b200.build``).
The functions below only marshal arguments: they check dtypes, devices and
shapes of torch tensors, allocate outputs when none are given, and pass raw
device pointers and the current CUDA stream to the library.  Every step of
the computation runs in the library's CUDA kernels; there is no fallback, and
every function raises if the library is missing or returns an error.

    codes, scales = kq_quantize(act, factors)            # [M, d/2], [M, d/32] uint8
    codes, scales = kq_quantize_shared(act, factors5)
    codes, scales = sq_quantize(act, mult)
    codes, scales = mx_quantize(act)
    W_folded      = kq_fold_weights(W, factors, shared=False)
    y             = kq_transform_f32(act, factors, shared=False)

W4A4 consumer (scales in the tensor core's scale-factor layout):

    codes, sf     = kq_quantize_sf(act, factors)         # [M, d/2], [kq_sf_bytes(M, d)] uint8
    wcodes, wsf   = mx_quantize_f32(W_folded, sf_layout=True)
    out           = mxf4_gemm(codes, sf, wcodes, wsf)    # bf16 [M, N] = X W^T, W4A4
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "LIB_PATH", "KQ_OK", "KQ_ERR_NULL", "KQ_ERR_SHAPE", "KQ_ERR_ALIGN", "KQ_ERR_CUDA", "KQ_ERR_VARIANT",
    "KroQuantError", "lib", "kq_quantize", "kq_quantize_shared", "kq_quantize_variant", "sq_quantize",
    "mx_quantize", "kq_fold_weights", "kq_transform_f32", "kq_last_error", "kq_abi_version",
    "sq_quantize_variant", "mx_quantize_variant", "kq_wait_timeouts", "kq_selftest_bounded_wait",
    "kq_transform_f32_variant", "kq_quantize_lu", "fwht_quantize", "kq_inverse_f32", "mx_dequantize", "norm_kq_quantize",
    "KQ_SCALES_ROWMAJOR", "KQ_SCALES_SF", "kq_sf_bytes", "kq_quantize_sf", "mx_quantize_f32", "mx_scales_to_sf",
    "mxf4_gemm", "mxf4_gemm_variant", "norm_kq_quantize_sf", "norm_kq_quantize_variant",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkroquant.so")

KQ_OK, KQ_ERR_NULL, KQ_ERR_SHAPE, KQ_ERR_ALIGN, KQ_ERR_CUDA, KQ_ERR_VARIANT = 0, -1, -2, -3, -4, -5
KQ_SCALES_ROWMAJOR, KQ_SCALES_SF = 0, 1

# Entry points and their argument types (p = pointer, i = int, q = int64).
_SIGS = {
    "kq_quantize": "ppppqqp",
    "kq_quantize_shared": "ppppqqp",
    "kq_quantize_variant": "ippippqqp",
    "sq_quantize_variant": "ippppqqp",
    "mx_quantize_variant": "ipppqqp",
    "kq_selftest_bounded_wait": "p",
    "sq_quantize": "ppppqqp",
    "mx_quantize": "pppqqp",
    "kq_fold_weights": "ppipqqp",
    "kq_transform_f32": "ppipqqp",
    "kq_transform_f32_variant": "ippipqqp",
    "kq_quantize_lu": "ppippqqp",
    "fwht_quantize": "pqppqqp",
    "kq_inverse_f32": "ppipqqp",
    "mx_dequantize": "pppqqp",
    "kq_quantize_sf": "ppippqqp",
    "mx_quantize_f32": "pppiqqp",
    "mx_scales_to_sf": "ppqqp",
    "mxf4_gemm": "pppppiqqqp",
    "mxf4_gemm_variant": "ipppppiqqqp",
}

_lib = None


class KroQuantError(RuntimeError):
    """A non-OK status from the library, with its status code and message."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"KroQuant CUDA library not found at {LIB_PATH}; build it with "
                "`python -m w4a4_mxfp4_post_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        kinds = {"p": ctypes.c_void_p, "i": ctypes.c_int, "q": ctypes.c_int64}
        for name, sig in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = [kinds[c] for c in sig]
            fn.restype = ctypes.c_int
        L.kq_last_error.argtypes = []
        L.kq_last_error.restype = ctypes.c_char_p
        L.kq_abi_version.argtypes = []
        L.kq_abi_version.restype = ctypes.c_int
        L.kq_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
        L.kq_wait_timeouts.restype = ctypes.c_int
        L.norm_kq_quantize.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_float, ctypes.c_void_p,
                                                                ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                                                ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.norm_kq_quantize.restype = ctypes.c_int
        L.norm_kq_quantize_sf.argtypes = L.norm_kq_quantize.argtypes
        L.norm_kq_quantize_sf.restype = ctypes.c_int
        L.norm_kq_quantize_variant.argtypes = [ctypes.c_int] + L.norm_kq_quantize.argtypes
        L.norm_kq_quantize_variant.restype = ctypes.c_int
        L.kq_sf_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        L.kq_sf_bytes.restype = ctypes.c_int64
        _lib = L
    return _lib


def kq_last_error() -> str:
    return lib().kq_last_error().decode()


def kq_abi_version() -> int:
    return lib().kq_abi_version()


def _call(name: str, device, *args) -> None:
    """Call entry point `name` with `device` (the tensors' device; None = the
    current one) as the current CUDA device: the library launches on the
    current device and caches its properties per device."""
    fn = getattr(lib(), name)
    if device is not None and device.index is not None and device.index != _torch().cuda.current_device():
        with _torch().cuda.device(device):
            rc = fn(*args)
    else:
        rc = fn(*args)
    if rc != KQ_OK:
        raise KroQuantError(name, rc, kq_last_error())


def _torch():
    import torch

    return torch


def _stream(stream, device):
    """The raw handle of `stream`, default the current stream of `device`; a
    torch stream must belong to `device`."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif isinstance(stream, torch.cuda.Stream) and device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr() if t is not None and t.numel() > 0 else 0)


def _need(t, name, dtype, device=None, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _act(act):
    torch = _torch()
    _need(act, "act", torch.bfloat16)
    if act.dim() != 2:
        raise ValueError("act must be 2-D [M, d]")
    return act.shape


def _outs(act, out_codes, out_scales):
    torch = _torch()
    M, d = act.shape
    if out_codes is None:
        out_codes = torch.empty((M, d // 2), dtype=torch.uint8, device=act.device)
    if out_scales is None:
        out_scales = torch.empty((M, d // 32), dtype=torch.uint8, device=act.device)
    _need(out_codes, "out_codes", torch.uint8, act.device, (M, d // 2))
    _need(out_scales, "out_scales", torch.uint8, act.device, (M, d // 32))
    return out_codes, out_scales


def _factors(factors, d, shared, device):
    torch = _torch()
    _need(factors, "factors", torch.float32, device)
    n = 1 if shared else d // 32
    if factors.numel() != n * 20:
        raise ValueError(f"factors must hold {n} x 5 x 2 x 2 floats, got {tuple(factors.shape)}")
    return factors


def kq_quantize(act, factors, out_codes=None, out_scales=None, stream=None):
    """KroQuant quantizer with one factor set per 32-column block ([d/32, 5, 2, 2])."""
    M, d = _act(act)
    _factors(factors, d, False, act.device)
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("kq_quantize", act.device, _ptr(act), _ptr(factors), _ptr(out_codes), _ptr(out_scales), M, d,
          _stream(stream, act.device))
    return out_codes, out_scales


def kq_quantize_shared(act, factors, out_codes=None, out_scales=None, stream=None):
    """KroQuant quantizer with one factor set ([5, 2, 2]) for every block."""
    M, d = _act(act)
    _factors(factors, d, True, act.device)
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("kq_quantize_shared", act.device, _ptr(act), _ptr(factors), _ptr(out_codes), _ptr(out_scales), M, d,
          _stream(stream, act.device))
    return out_codes, out_scales


def kq_quantize_variant(variant, act, factors, shared=False, out_codes=None, out_scales=None, stream=None):
    """The KroQuant quantizer through a chosen kernel variant (0 = the default)."""
    M, d = _act(act)
    _factors(factors, d, shared, act.device)
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("kq_quantize_variant", act.device, int(variant), _ptr(act), _ptr(factors), int(bool(shared)), _ptr(out_codes),
          _ptr(out_scales), M, d, _stream(stream, act.device))
    return out_codes, out_scales


def sq_quantize(act, mult, out_codes=None, out_scales=None, stream=None):
    """SmoothQuant baseline: fp32(x * mult[c]) per channel, then MXFP4."""
    torch = _torch()
    M, d = _act(act)
    _need(mult, "mult", torch.float32, act.device, (d,))
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("sq_quantize", act.device, _ptr(act), _ptr(mult), _ptr(out_codes), _ptr(out_scales), M, d,
          _stream(stream, act.device))
    return out_codes, out_scales


def mx_quantize(act, out_codes=None, out_scales=None, stream=None):
    """Plain MXFP4 baseline (no transform)."""
    M, d = _act(act)
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("mx_quantize", act.device, _ptr(act), _ptr(out_codes), _ptr(out_scales), M, d, _stream(stream, act.device))
    return out_codes, out_scales


def kq_quantize_lu(act, lu_params, shared=False, out_codes=None, out_scales=None, stream=None):
    """KroQuant quantizer from 15 LU scalars per block ([d/32, 5, 3] or [5, 3] if shared)."""
    torch = _torch()
    M, d = _act(act)
    _need(lu_params, "lu_params", torch.float32, act.device)
    n = 1 if shared else d // 32
    if lu_params.numel() != n * 15:
        raise ValueError(f"lu_params must hold {n} x 5 x 3 floats, got {tuple(lu_params.shape)}")
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("kq_quantize_lu", act.device, _ptr(act), _ptr(lu_params), int(bool(shared)), _ptr(out_codes),
          _ptr(out_scales), M, d, _stream(stream, act.device))
    return out_codes, out_scales


def fwht_quantize(act, H, out_codes=None, out_scales=None, stream=None):
    """Fixed-Hadamard (block size H) baseline quantizer."""
    M, d = _act(act)
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("fwht_quantize", act.device, _ptr(act), int(H), _ptr(out_codes), _ptr(out_scales), M, d,
          _stream(stream, act.device))
    return out_codes, out_scales


def norm_kq_quantize(h, gamma, beta, factors, eps=1e-6, shared=False, out_codes=None, out_scales=None,
                     stream=None):
    """LayerNorm + AdaLN modulation (gamma, beta: [nsamples, d]) fused with kq_quantize."""
    return norm_kq_quantize_variant(0, h, gamma, beta, factors, eps, shared, out_codes, out_scales, stream)


def norm_kq_quantize_variant(variant, h, gamma, beta, factors, eps=1e-6, shared=False, out_codes=None,
                             out_scales=None, stream=None):
    """norm_kq_quantize through a chosen kernel (0 = the default)."""
    torch = _torch()
    M, d = _act(h)
    _need(gamma, "gamma", torch.float32, h.device)
    _need(beta, "beta", torch.float32, h.device, tuple(gamma.shape))
    if gamma.dim() != 2 or gamma.shape[1] != d:
        raise ValueError("gamma and beta must be [nsamples, d]")
    _factors(factors, d, shared, h.device)
    out_codes, out_scales = _outs(h, out_codes, out_scales)
    args = (_ptr(h), _ptr(gamma), _ptr(beta), int(gamma.shape[0]), float(eps), _ptr(factors), int(bool(shared)),
            _ptr(out_codes), _ptr(out_scales), M, d, _stream(stream, h.device))
    if variant == 0:
        _call("norm_kq_quantize", h.device, *args)
    else:
        _call("norm_kq_quantize_variant", h.device, int(variant), *args)
    return out_codes, out_scales


def kq_inverse_f32(y, factors, shared=False, out=None, stream=None):
    """x = T^-1 y per 32-block (fp32 [M, d])."""
    torch = _torch()
    _need(y, "y", torch.float32)
    if y.dim() != 2:
        raise ValueError("y must be 2-D [M, d]")
    M, d = y.shape
    _factors(factors, d, shared, y.device)
    if out is None:
        out = torch.empty_like(y)
    _need(out, "out", torch.float32, y.device, (M, d))
    _call("kq_inverse_f32", y.device, _ptr(y), _ptr(factors), int(bool(shared)), _ptr(out), M, d,
          _stream(stream, y.device))
    return out


def mx_dequantize(codes, scales, out=None, stream=None):
    """MXFP4 decode of codes [M, d/2] and scales [M, d/32] to fp32 [M, d]."""
    torch = _torch()
    _need(codes, "codes", torch.uint8)
    if codes.dim() != 2:
        raise ValueError("codes must be 2-D [M, d/2]")
    M, d = codes.shape[0], codes.shape[1] * 2
    _need(scales, "scales", torch.uint8, codes.device, (M, d // 32))
    if out is None:
        out = torch.empty((M, d), dtype=torch.float32, device=codes.device)
    _need(out, "out", torch.float32, codes.device, (M, d))
    _call("mx_dequantize", codes.device, _ptr(codes), _ptr(scales), _ptr(out), M, d, _stream(stream, codes.device))
    return out


def sq_quantize_variant(variant, act, mult, out_codes=None, out_scales=None, stream=None):
    """The SmoothQuant quantizer through a chosen kernel variant (0 = the default)."""
    torch = _torch()
    M, d = _act(act)
    _need(mult, "mult", torch.float32, act.device, (d,))
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("sq_quantize_variant", act.device, int(variant), _ptr(act), _ptr(mult), _ptr(out_codes), _ptr(out_scales), M,
          d, _stream(stream, act.device))
    return out_codes, out_scales


def mx_quantize_variant(variant, act, out_codes=None, out_scales=None, stream=None):
    """The plain MXFP4 quantizer through a chosen kernel variant (0 = the default)."""
    M, d = _act(act)
    out_codes, out_scales = _outs(act, out_codes, out_scales)
    _call("mx_quantize_variant", act.device, int(variant), _ptr(act), _ptr(out_codes), _ptr(out_scales), M, d,
          _stream(stream, act.device))
    return out_codes, out_scales


def kq_wait_timeouts(reset: bool = False) -> int:
    """Number of bounded waits that gave up in the staged kernels (synchronises the device)."""
    v = ctypes.c_int(0)
    rc = lib().kq_wait_timeouts(ctypes.byref(v), int(bool(reset)))
    if rc != KQ_OK:
        raise KroQuantError("kq_wait_timeouts", rc, kq_last_error())
    return v.value


def kq_selftest_bounded_wait(stream=None) -> None:
    """Launch one staged CTA whose waits run out (no copies issued); see the C header."""
    _call("kq_selftest_bounded_wait", None, _stream(stream, None))


def kq_fold_weights(W, factors, shared=False, out=None, stream=None):
    """W T^-1 per 32-column block (fp32 [N, d])."""
    torch = _torch()
    _need(W, "W", torch.float32)
    if W.dim() != 2:
        raise ValueError("W must be 2-D [N, d]")
    N, d = W.shape
    _factors(factors, d, shared, W.device)
    if out is None:
        out = torch.empty_like(W)
    _need(out, "out", torch.float32, W.device, (N, d))
    _call("kq_fold_weights", W.device, _ptr(W), _ptr(factors), int(bool(shared)), _ptr(out), N, d,
          _stream(stream, W.device))
    return out


def kq_transform_f32_variant(variant, act, factors, shared=False, out=None, stream=None):
    """The fp32 transform through a chosen kernel variant (test export)."""
    torch = _torch()
    M, d = _act(act)
    _factors(factors, d, shared, act.device)
    if out is None:
        out = torch.empty((M, d), dtype=torch.float32, device=act.device)
    _need(out, "out", torch.float32, act.device, (M, d))
    _call("kq_transform_f32_variant", act.device, int(variant), _ptr(act), _ptr(factors), int(bool(shared)), _ptr(out),
          M, d, _stream(stream, act.device))
    return out


def kq_transform_f32(act, factors, shared=False, out=None, stream=None):
    """The fp32 transform y = T x that the quantizer computes (test export)."""
    torch = _torch()
    M, d = _act(act)
    _factors(factors, d, shared, act.device)
    if out is None:
        out = torch.empty((M, d), dtype=torch.float32, device=act.device)
    _need(out, "out", torch.float32, act.device, (M, d))
    _call("kq_transform_f32", act.device, _ptr(act), _ptr(factors), int(bool(shared)), _ptr(out), M, d,
          _stream(stream, act.device))
    return out


def kq_sf_bytes(rows: int, d: int) -> int:
    """Bytes of a scale-factor-layout buffer for a [rows, d] MXFP4 matrix."""
    n = lib().kq_sf_bytes(int(rows), int(d))
    if n < 0:
        raise ValueError(f"kq_sf_bytes: bad shape rows={rows}, d={d}")
    return n


def _sf_out(out_sf, rows, d, device):
    torch = _torch()
    n = kq_sf_bytes(rows, d)
    if out_sf is None:
        out_sf = torch.empty((n,), dtype=torch.uint8, device=device)
    _need(out_sf, "out_sf", torch.uint8, device, (n,))
    return out_sf


def kq_quantize_sf(act, factors, shared=False, out_codes=None, out_sf=None, stream=None):
    """kq_quantize with the scales in the tensor core's scale-factor layout (1-D uint8)."""
    torch = _torch()
    M, d = _act(act)
    _factors(factors, d, shared, act.device)
    if out_codes is None:
        out_codes = torch.empty((M, d // 2), dtype=torch.uint8, device=act.device)
    _need(out_codes, "out_codes", torch.uint8, act.device, (M, d // 2))
    out_sf = _sf_out(out_sf, M, d, act.device)
    _call("kq_quantize_sf", act.device, _ptr(act), _ptr(factors), int(bool(shared)), _ptr(out_codes), _ptr(out_sf), M,
          d, _stream(stream, act.device))
    return out_codes, out_sf


def mx_quantize_f32(x, sf_layout=False, out_codes=None, out_scales=None, stream=None):
    """Plain MXFP4 quantizer on fp32 input [M, d] (the folded weights).

    Scales row-major [M, d/32], or with sf_layout=True in the scale-factor layout (1-D).
    """
    torch = _torch()
    _need(x, "x", torch.float32)
    if x.dim() != 2:
        raise ValueError("x must be 2-D [M, d]")
    M, d = x.shape
    if out_codes is None:
        out_codes = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    _need(out_codes, "out_codes", torch.uint8, x.device, (M, d // 2))
    if sf_layout:
        out_scales = _sf_out(out_scales, M, d, x.device)
    else:
        if out_scales is None:
            out_scales = torch.empty((M, d // 32), dtype=torch.uint8, device=x.device)
        _need(out_scales, "out_scales", torch.uint8, x.device, (M, d // 32))
    _call("mx_quantize_f32", x.device, _ptr(x), _ptr(out_codes), _ptr(out_scales),
          KQ_SCALES_SF if sf_layout else KQ_SCALES_ROWMAJOR, M, d, _stream(stream, x.device))
    return out_codes, out_scales


def mx_scales_to_sf(scales, out_sf=None, stream=None):
    """Row-major scales [M, d/32] -> the scale-factor layout (1-D uint8)."""
    torch = _torch()
    _need(scales, "scales", torch.uint8)
    if scales.dim() != 2:
        raise ValueError("scales must be 2-D [M, d/32]")
    M, d = scales.shape[0], scales.shape[1] * 32
    out_sf = _sf_out(out_sf, M, d, scales.device)
    _call("mx_scales_to_sf", scales.device, _ptr(scales), _ptr(out_sf), M, d, _stream(stream, scales.device))
    return out_sf


def mxf4_gemm(a_codes, a_sf, b_codes, b_sf, out=None, out_dtype=None, stream=None):
    """W4A4 linear layer: out[m, n] = sum_k a[m, k] b[n, k] over decoded MXFP4 operands.

    a_codes [M, K/2], b_codes [N, K/2] uint8; a_sf, b_sf their scales in the
    scale-factor layout; out bf16 (default) or float32 [M, N].
    """
    return mxf4_gemm_variant(0, a_codes, a_sf, b_codes, b_sf, out, out_dtype, stream)


def mxf4_gemm_variant(variant, a_codes, a_sf, b_codes, b_sf, out=None, out_dtype=None, stream=None):
    """mxf4_gemm through a chosen tile configuration (0 = the default; test export)."""
    torch = _torch()
    _need(a_codes, "a_codes", torch.uint8)
    if a_codes.dim() != 2 or b_codes.dim() != 2:
        raise ValueError("a_codes and b_codes must be 2-D")
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    dev = a_codes.device
    _need(b_codes, "b_codes", torch.uint8, dev)
    N = b_codes.shape[0]
    if b_codes.shape[1] * 2 != K:
        raise ValueError(f"b_codes must be [N, {K // 2}], got {tuple(b_codes.shape)}")
    _need(a_sf, "a_sf", torch.uint8, dev, (kq_sf_bytes(M, K),))
    _need(b_sf, "b_sf", torch.uint8, dev, (kq_sf_bytes(N, K),))
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=dev)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, dev, (M, N))
    _call("mxf4_gemm_variant", dev, int(variant), _ptr(a_codes), _ptr(a_sf), _ptr(b_codes), _ptr(b_sf), _ptr(out),
          int(out.dtype == torch.float32), M, N, K, _stream(stream, dev))
    return out


def norm_kq_quantize_sf(h, gamma, beta, factors, eps=1e-6, shared=False, out_codes=None, out_sf=None, stream=None):
    """norm_kq_quantize with the scales in the tensor core's scale-factor layout (1-D uint8)."""
    torch = _torch()
    M, d = _act(h)
    _need(gamma, "gamma", torch.float32, h.device)
    _need(beta, "beta", torch.float32, h.device, tuple(gamma.shape))
    if gamma.dim() != 2 or gamma.shape[1] != d:
        raise ValueError("gamma and beta must be [nsamples, d]")
    _factors(factors, d, shared, h.device)
    if out_codes is None:
        out_codes = torch.empty((M, d // 2), dtype=torch.uint8, device=h.device)
    _need(out_codes, "out_codes", torch.uint8, h.device, (M, d // 2))
    out_sf = _sf_out(out_sf, M, d, h.device)
    _call("norm_kq_quantize_sf", h.device, _ptr(h), _ptr(gamma), _ptr(beta), int(gamma.shape[0]), float(eps),
          _ptr(factors), int(bool(shared)), _ptr(out_codes), _ptr(out_sf), M, d, _stream(stream, h.device))
    return out_codes, out_sf
