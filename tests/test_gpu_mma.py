"""The tensor-core (tcgen05) KroQuant variant against the oracle."""
import numpy as np
import pytest

import oracle
import parity_check as pc
import w4a4_mxfp4_post_b200 as kq
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu

MMAS = (4,)


def dev_bf16(bits, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev_f32(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


# small first: one tile, one partial column group, a single block, ragged rows
SHAPES = [(1, 32), (128, 128), (3, 96), (130, 160), (37, 64), (129, 5600), (257, 2240), (1000, 1152),
          (300, 12288), (8192, 4608)]


@pytest.mark.parametrize("MMA", MMAS)
@pytest.mark.parametrize("M,d", SHAPES, ids=[f"{M}x{d}" for M, d in SHAPES])
def test_mma_variant_matches_oracle(cuda_device, M, d, MMA):
    x = synth.activation("pixart", M, d, seed=M * 5 + d)
    F = synth.factors(d // 32, seed=d + 2)
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    kq.kq_wait_timeouts(reset=True)
    c, s = kq.kq_quantize_variant(MMA, xd, Fd)
    y = kq.kq_transform_f32_variant(MMA, xd, Fd).cpu().numpy()
    assert kq.kq_wait_timeouts() == 0
    cr, sr = oracle.kq_quantize(x, F)
    yr, ab = oracle.kq_transform(x, F, want_absbound=True)
    tr = pc.check_transform(y, yr, ab)
    assert tr["bad"] == 0, tr
    res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
    assert res["ok"], res


@pytest.mark.parametrize("MMA", MMAS)
def test_mma_variant_shared_factors(cuda_device, MMA):
    M, d = 300, 2240
    x = synth.activation("sana", M, d, 2)
    F1 = synth.factors(1, 2, shared=True)
    xd = dev_bf16(x, cuda_device)
    c, s = kq.kq_quantize_variant(MMA, xd, dev_f32(F1, cuda_device), shared=True)
    cr, sr = oracle.kq_quantize(x, F1, shared=True)
    yr, ab = oracle.kq_transform(x, F1, shared=True, want_absbound=True)
    res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
    assert res["ok"], res


@pytest.mark.parametrize("MMA", MMAS)
def test_mma_variant_hand_worked_blocks(cuda_device, MMA):
    import os

    from conftest import GOLDEN, parse_blocks

    for case in parse_blocks(os.path.join(GOLDEN, "hand_blocks.txt")):
        x = dev_bf16(synth.bf16_bits_from_f32(case["x"]), cuda_device)
        c, s = kq.kq_quantize_variant(MMA, x, dev_f32(case["factors"], cuda_device))
        assert int(s.cpu()[0, 0]) == case["scale"], case["name"]
        np.testing.assert_array_equal(c.cpu().numpy()[0], case["codes"], err_msg=case["name"])
