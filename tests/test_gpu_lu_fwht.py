"""The LU-parametrised KroQuant quantizer and the fixed-Hadamard (FWHT) baseline vs the oracle."""
import numpy as np
import pytest

import oracle
import parity_check as pc
import w4a4_mxfp4_post_b200 as kq
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu


def dev_bf16(bits, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev_f32(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


LU_SHAPES = [(1, 32), (37, 96), (257, 2240), (129, 5600), (8192, 4608)]


@pytest.mark.parametrize("M,d", LU_SHAPES, ids=[f"{M}x{d}" for M, d in LU_SHAPES])
def test_lu_quantizer_matches_oracle(cuda_device, M, d):
    x = synth.activation("pixart", M, d, seed=M + 3 * d)
    P = synth.lu_params(d // 32, seed=d)
    c, s = kq.kq_quantize_lu(dev_bf16(x, cuda_device), dev_f32(P, cuda_device))
    cr, sr = oracle.kq_quantize_lu(x, P)
    yr, ab = oracle.kq_transform_lu(x, P, want_absbound=True)
    res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
    assert res["ok"], res


def test_lu_quantizer_shared_and_hadamard_init(cuda_device):
    M, d = 300, 2240
    x = synth.activation("sana", M, d, 2)
    for P in (synth.lu_params(1, 5, shared=True),
              np.tile(np.array([1 / np.sqrt(2.0), 1 / np.sqrt(2.0), 1.0], np.float32), (1, 5, 1))):
        c, s = kq.kq_quantize_lu(dev_bf16(x, cuda_device), dev_f32(P, cuda_device), shared=True)
        cr, sr = oracle.kq_quantize_lu(x, P, shared=True)
        yr, ab = oracle.kq_transform_lu(x, P, shared=True, want_absbound=True)
        res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
        assert res["ok"], res


FWHT_CASES = [(37, 1024, 32), (37, 1024, 64), (64, 1024, 128), (64, 1024, 256), (33, 1024, 512),
              (33, 1024, 1024), (8192, 4608, 512), (8192, 1152, 128), (300, 3072, 1024)]


@pytest.mark.parametrize("M,d,H", FWHT_CASES, ids=[f"{M}x{d}-H{H}" for M, d, H in FWHT_CASES])
def test_fwht_quantizer_matches_oracle(cuda_device, M, d, H):
    x = synth.activation("pixart", M, d, seed=H + M)
    c, s = kq.fwht_quantize(dev_bf16(x, cuda_device), H)
    cr, sr = oracle.fwht_quantize(x, H)
    yr, ab = oracle.fwht_transform(x, H, want_absbound=True)
    res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
    assert res["ok"], (H, res)


def test_fwht_shape_errors(cuda_device):
    x = dev_bf16(synth.activation("pixart", 4, 96, 1), cuda_device)
    for H in (16, 48, 2048):
        with pytest.raises(kq.KroQuantError) as ei:
            kq.fwht_quantize(x, H)
        assert ei.value.status == kq.KQ_ERR_SHAPE
    with pytest.raises(kq.KroQuantError) as ei:
        kq.fwht_quantize(x, 64)           # 96 % 64 != 0
    assert ei.value.status == kq.KQ_ERR_SHAPE
