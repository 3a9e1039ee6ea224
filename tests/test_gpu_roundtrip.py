"""MXFP4 decode and the inverse transform (the round trip x -> codes -> x^) vs the oracle."""
import numpy as np
import pytest

import oracle
import w4a4_mxfp4_post_b200 as kq
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu


def dev(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def test_dequantize_is_exact(cuda_device):
    rng = np.random.default_rng(41)
    M, d = 257, 1152
    codes = rng.integers(0, 256, (M, d // 2), dtype=np.uint8)
    scales = rng.integers(0, 255, (M, d // 32), dtype=np.uint8)
    scales[0, :3] = (0, 1, 254)
    out = kq.mx_dequantize(dev(codes, cuda_device), dev(scales, cuda_device)).cpu().numpy()
    np.testing.assert_array_equal(out, oracle.mx_dequantize(codes, scales))
    scales[1, 0] = 0xFF
    out = kq.mx_dequantize(dev(codes, cuda_device), dev(scales, cuda_device)).cpu().numpy()
    assert np.isnan(out[1, :32]).all()


@pytest.mark.parametrize("M,d,shared", [(64, 128, False), (1000, 4608, False), (33, 2240, True)])
def test_inverse_matches_oracle(cuda_device, M, d, shared):
    import torch

    rng = np.random.default_rng(M + d)
    y = (rng.standard_normal((M, d)) * 5).astype(np.float32)
    F = synth.factors(d // 32, seed=d, shared=shared)
    x = kq.kq_inverse_f32(dev(y, cuda_device), dev(F, cuda_device), shared=shared).cpu().numpy()
    xr, ab = oracle.kq_inverse(y, F, shared=shared, want_absbound=True)
    np.testing.assert_array_less(np.abs(x.astype(np.float64) - xr), 1e-5 * ab + 1e-30)
    del torch


def test_round_trip_matches_oracle_error(cuda_device):
    M, d = 2048, 1152
    x = synth.activation("pixart", M, d, 42)
    F = synth.factors(d // 32, 42)
    xd, Fd = dev(x.view(np.int16), cuda_device), dev(F, cuda_device)
    import torch

    xd = xd.view(torch.bfloat16)
    c, s = kq.kq_quantize(xd, Fd)
    xh = kq.kq_inverse_f32(kq.mx_dequantize(c, s), Fd).cpu().numpy().astype(np.float64)
    cr, sr = oracle.kq_quantize(x, F)
    xhr = oracle.kq_inverse(oracle.mx_dequantize(cr, sr), F).astype(np.float64)
    xv = synth.bf16_bits_to_f32(x).astype(np.float64)
    e_gpu = np.sum((xv - xh) ** 2)
    e_ref = np.sum((xv - xhr) ** 2)
    assert abs(e_gpu / e_ref - 1) < 1e-3, (e_gpu, e_ref)
