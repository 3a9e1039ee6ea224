"""The quantizer fused with LayerNorm + AdaLN modulation vs the oracle."""
import numpy as np
import pytest

import oracle
import parity_check as pc
import w4a4_mxfp4_post_b200 as kq
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu

EPS = 1e-6
NORM_VARIANTS = (0, 1, 2, 3)


def dev(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def dev_bf16(bits, device):
    import torch

    return dev(bits.view(np.int16), device).view(torch.bfloat16)


CASES = [(64, 128, 1, False), (37, 96, 1, False), (8192, 1152, 2, False), (2048, 5600, 2, False), (1000, 4608, 4, False),
         (2048, 2240, 4, True), (512, 12288, 2, False), (300, 4608, 3, False)]


@pytest.mark.parametrize("M,d,ns,shared", CASES, ids=[f"{c[0]}x{c[1]}-s{c[2]}{'-shared' if c[3] else ''}"
                                                       for c in CASES])
def test_norm_kq_matches_oracle(cuda_device, M, d, ns, shared):
    h = synth.activation("pixart", M, d, seed=M + d)
    gamma, beta = synth.adaln(ns, d, seed=d)
    F = synth.factors(d // 32, seed=d, shared=shared)
    ref = oracle.norm_kq(h, gamma, beta, EPS, F, shared=shared, want=("codes", "y", "absb"))
    args = (dev_bf16(h, cuda_device), dev(gamma, cuda_device), dev(beta, cuda_device), dev(F, cuda_device))
    # the default and each of the three kernels (row buffers, row re-read, one CTA per row)
    for v in NORM_VARIANTS:
        c, s = kq.norm_kq_quantize_variant(v, *args, eps=EPS, shared=shared)
        res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), ref["codes"], ref["scales"], ref["y"], ref["absb"])
        assert res["ok"], (v, res)


def test_norm_kq_shape_errors(cuda_device):
    import torch

    h = dev_bf16(synth.activation("pixart", 6, 64, 1), cuda_device)
    g = torch.zeros((4, 64), dtype=torch.float32, device=cuda_device)
    F = dev(synth.factors(2, 1), cuda_device)
    with pytest.raises(kq.KroQuantError) as ei:          # 6 rows, 4 samples
        kq.norm_kq_quantize(h, g, g.clone(), F)
    assert ei.value.status == kq.KQ_ERR_SHAPE


@pytest.mark.parametrize("M,d,ns", [(300, 4608, 3), (129, 96, 1), (512, 12288, 2), (2048, 5600, 2)])
def test_norm_kq_sf_layout_matches_row_major_path(cuda_device, M, d, ns):
    """Same codes as norm_kq_quantize; the scales are its row-major scales in the
    oracle's scale-factor layout, including the odd-block pad (whole buffer,
    pre-filled with 0xFF, compared)."""
    import torch

    h = synth.activation("pixart", M, d, seed=M + 2 * d)
    gamma, beta = synth.adaln(ns, d, seed=d + 1)
    F = synth.factors(d // 32, seed=d + 2)
    args = (dev_bf16(h, cuda_device), dev(gamma, cuda_device), dev(beta, cuda_device), dev(F, cuda_device))
    c, s = kq.norm_kq_quantize(*args, eps=EPS)
    sf0 = torch.full((kq.kq_sf_bytes(M, d),), 0xFF, dtype=torch.uint8, device=cuda_device)
    c2, sf = kq.norm_kq_quantize_sf(*args, eps=EPS, out_sf=sf0)
    np.testing.assert_array_equal(c2.cpu().numpy(), c.cpu().numpy())
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.scales_to_sf(s.cpu().numpy()))


@pytest.mark.parametrize("M,d", [(256, 1152), (300, 4608), (64, 12288)])
def test_norm_kq_large_mean_takes_the_two_pass_variance(cuda_device, M, d):
    """Rows whose mean is large against their spread (each row shifted by half
    its root mean square, so mu^2 > E[x^2] / 64): the one-sweep variance
    E[x^2] - mu^2 is not used there and the kernel takes the two-pass form; the
    result meets the oracle criteria.  (A mean far above the spread, with the
    spread near bf16's resolution, would be ill-conditioned for any fp32
    LayerNorm: the mean's rounding is amplified by 1 / sigma.)"""
    x = synth.bf16_bits_to_f32(synth.activation("pixart", M, d, seed=7)).astype(np.float64)
    rms = np.sqrt((x * x).mean(axis=1, keepdims=True))
    h = synth.bf16_bits_from_f32((x + 0.5 * rms).astype(np.float32))
    hv = synth.bf16_bits_to_f32(h).astype(np.float64)
    assert np.all(hv.mean(axis=1) ** 2 > (hv * hv).mean(axis=1) / 64)     # the two-pass branch
    gamma, beta = synth.adaln(2, d, seed=d)
    F = synth.factors(d // 32, seed=d)
    ref = oracle.norm_kq(h, gamma, beta, EPS, F, want=("codes", "y", "absb"))
    args = (dev_bf16(h, cuda_device), dev(gamma, cuda_device), dev(beta, cuda_device), dev(F, cuda_device))
    for v in NORM_VARIANTS:
        c, s = kq.norm_kq_quantize_variant(v, *args, eps=EPS)
        res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), ref["codes"], ref["scales"], ref["y"], ref["absb"])
        assert res["ok"], (v, res)


def test_norm_kq_variant_errors(cuda_device):
    h = dev_bf16(synth.activation("pixart", 4, 64, 1), cuda_device)
    g = dev(np.zeros((1, 64), np.float32), cuda_device)
    F = dev(synth.factors(2, 1), cuda_device)
    with pytest.raises(kq.KroQuantError) as ei:
        kq.norm_kq_quantize_variant(4, h, g, g.clone(), F)
    assert ei.value.status == kq.KQ_ERR_VARIANT
