"""Edge cases, cross-kernel identities and error paths of the CUDA path."""
import os

import numpy as np
import pytest

import oracle
import parity_check as pc
import w4a4_mxfp4_post_b200 as kq
from conftest import GOLDEN, parse_blocks
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu

CANARY = 0xA5


def dev_bf16(bits, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev_f32(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def guarded(shape, device, pad=256):
    """A uint8 output view followed by `pad` canary bytes in the same allocation."""
    import torch

    n = int(np.prod(shape))
    buf = torch.full((n + pad,), CANARY, dtype=torch.uint8, device=device)
    return buf, buf[:n].view(*shape)


def bf16(a):
    return synth.bf16_bits_from_f32(np.asarray(a, np.float32))


@pytest.mark.parametrize("case", parse_blocks(os.path.join(GOLDEN, "hand_blocks.txt")), ids=lambda c: c["name"])
def test_hand_worked_blocks_on_gpu(cuda_device, case):
    x = dev_bf16(bf16(case["x"]), cuda_device)
    F = dev_f32(case["factors"], cuda_device)
    c, s = kq.kq_quantize(x, F)
    assert int(s.cpu()[0, 0]) == case["scale"]
    np.testing.assert_array_equal(c.cpu().numpy()[0], case["codes"])
    # the same blocks through the plain MX kernel when the factors are the identity
    if np.array_equal(case["factors"].reshape(5, 2, 2), np.tile(np.eye(2, dtype=np.float32), (5, 1, 1))):
        c2, s2 = kq.mx_quantize(x)
        np.testing.assert_array_equal(c2.cpu().numpy()[0], case["codes"])
        assert int(s2.cpu()[0, 0]) == case["scale"]


def test_exact_zeros_come_out_positive(cuda_device):
    """An exactly cancelling sum is +0 (as in the oracle), whichever form the kernel uses."""
    H = np.array([[1, 1], [1, -1]], np.float32)           # unit-diagonal split with D = diag(1, -1)
    S = np.array([[0, 1], [1, 0]], np.float32)            # no split: the direct form
    for F in (np.stack([H] * 5), np.stack([H, H, S, H, H])):
        xb = bf16(np.ones((1, 32), np.float32))
        y = kq.kq_transform_f32(dev_bf16(xb, cuda_device), dev_f32(F[None], cuda_device)).cpu().numpy()[0]
        yr = oracle.kq_transform(xb, F[None])[0]
        np.testing.assert_array_equal(y, yr)
        zeros = yr == 0
        assert zeros.sum() >= 30
        assert not np.signbit(y[zeros]).any() and not np.signbit(yr[zeros]).any()


RAGGED = [(1, 32), (3, 32), (37, 64), (5, 1152), (129, 5600), (7, 2240), (1000, 96), (2049, 160)]


@pytest.mark.parametrize("M,d", RAGGED, ids=[f"{M}x{d}" for M, d in RAGGED])
def test_ragged_shapes_and_canaries(cuda_device, M, d):
    x = synth.activation("pixart", M, d, seed=M + d)
    F = synth.factors(d // 32, seed=d)
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    cbuf, codes = guarded((M, d // 2), cuda_device)
    sbuf, scales = guarded((M, d // 32), cuda_device)
    kq.kq_quantize(xd, Fd, codes, scales)
    cb, sb = cbuf.cpu().numpy(), sbuf.cpu().numpy()
    assert np.all(cb[M * d // 2:] == CANARY) and np.all(sb[M * d // 32:] == CANARY)
    cr, sr = oracle.kq_quantize(x, F)
    yr, ab = oracle.kq_transform(x, F, want_absbound=True)
    res = pc.check_kq(cb[:M * d // 2].reshape(M, -1), sb[:M * d // 32].reshape(M, -1), cr, sr, yr, ab)
    assert res["ok"], res
    for fn, ref in ((lambda c, s: kq.mx_quantize(xd, c, s), oracle.mx_quantize(x)),
                    (lambda c, s: kq.sq_quantize(xd, dev_f32(np.full(d, 0.37, np.float32), cuda_device), c, s),
                     oracle.sq_quantize(x, np.full(d, 0.37, np.float32)))):
        cbuf, codes = guarded((M, d // 2), cuda_device)
        sbuf, scales = guarded((M, d // 32), cuda_device)
        fn(codes, scales)
        cb, sb = cbuf.cpu().numpy(), sbuf.cpu().numpy()
        assert np.all(cb[M * d // 2:] == CANARY) and np.all(sb[M * d // 32:] == CANARY)
        assert pc.check_exact(cb[:M * d // 2].reshape(M, -1), sb[:M * d // 32].reshape(M, -1), *ref)["ok"]


def test_transform_canary(cuda_device):
    import torch

    M, d = 33, 96
    x = synth.activation("tiny", M, d, 1)
    F = synth.factors(d // 32, 1)
    buf = torch.full((M * d + 64,), 7.0, dtype=torch.float32, device=cuda_device)
    kq.kq_transform_f32(dev_bf16(x, cuda_device), dev_f32(F, cuda_device), out=buf[:M * d].view(M, d))
    assert bool((buf[M * d:] == 7.0).all())


def test_identity_factors_equal_mx(cuda_device):
    M, d = 300, 1152
    x = dev_bf16(synth.activation("pixart", M, d, 21), cuda_device)
    I = dev_f32(np.tile(np.eye(2, dtype=np.float32), (d // 32, 5, 1, 1)), cuda_device)
    c1, s1 = kq.kq_quantize(x, I)
    c2, s2 = kq.mx_quantize(x)
    assert bool((c1 == c2).all()) and bool((s1 == s2).all())


def test_unit_multiplier_sq_equals_mx(cuda_device):
    import torch

    M, d = 300, 1152
    x = dev_bf16(synth.activation("pixart", M, d, 22), cuda_device)
    c1, s1 = kq.sq_quantize(x, torch.ones(d, dtype=torch.float32, device=cuda_device))
    c2, s2 = kq.mx_quantize(x)
    assert bool((c1 == c2).all()) and bool((s1 == s2).all())


def test_power_of_two_diagonal_factors_equal_mx_of_scaled_input(cuda_device):
    M, d = 64, 64
    x = synth.activation("pixart", M, d, 23)
    ex = np.array([[1, -2], [0, 3], [2, 0], [-1, 1], [0, 0]])
    F = np.stack([np.diag(2.0 ** e).astype(np.float32) for e in ex])
    sc = np.array([2.0 ** sum(ex[k][(i >> (4 - k)) & 1] for k in range(5)) for i in range(32)], np.float32)
    xs = bf16(synth.bf16_bits_to_f32(x) * np.tile(sc, d // 32)[None, :])
    c1, s1 = kq.kq_quantize(dev_bf16(x, cuda_device), dev_f32(np.stack([F] * (d // 32)), cuda_device))
    c2, s2 = kq.mx_quantize(dev_bf16(xs, cuda_device))
    assert bool((c1 == c2).all()) and bool((s1 == s2).all())


def test_swap_factors_equal_mx_of_bit_permuted_input(cuda_device):
    # A swap factor on bit b maps element i to position i ^ (1 << b).
    M, d = 64, 128
    x = synth.activation("pixart", M, d, 24)
    I2 = np.eye(2, dtype=np.float32)
    S = np.array([[0, 1], [1, 0]], np.float32)
    for k in range(5):
        F = np.stack([S if q == k else I2 for q in range(5)])
        bit = 4 - k
        perm = np.array([i ^ (1 << bit) for i in range(32)])
        xp = x.reshape(M, d // 32, 32)[:, :, perm].reshape(M, d)
        c1, s1 = kq.kq_quantize(dev_bf16(x, cuda_device), dev_f32(np.stack([F] * (d // 32)), cuda_device))
        c2, s2 = kq.mx_quantize(dev_bf16(xp, cuda_device))
        assert bool((c1 == c2).all()) and bool((s1 == s2).all()), k


def test_shared_equals_repeated_factors(cuda_device):
    M, d = 257, 2240
    x = dev_bf16(synth.activation("sana", M, d, 2), cuda_device)
    F1 = synth.factors(1, 2, shared=True)
    c1, s1 = kq.kq_quantize_shared(x, dev_f32(F1, cuda_device))
    c2, s2 = kq.kq_quantize(x, dev_f32(np.repeat(F1, d // 32, axis=0), cuda_device))
    assert bool((c1 == c2).all()) and bool((s1 == s2).all())


def test_variants_agree_with_oracle(cuda_device):
    M, d = 512, 3072
    x = synth.activation("flux", M, d, 3)
    F = synth.factors(d // 32, 3)
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    cr, sr = oracle.kq_quantize(x, F)
    yr, ab = oracle.kq_transform(x, F, want_absbound=True)
    tried = 0
    for v in range(10):
        try:
            c, s = kq.kq_quantize_variant(v, xd, Fd)
        except kq.KroQuantError as e:
            assert e.status == kq.KQ_ERR_VARIANT
            continue
        tried += 1
        res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
        assert res["ok"], (v, res)
    assert tried >= 1


# ragged final stage, odd block counts, a single block; 4099 x 1152 gives the
# two-block ring kernel an odd number of chunks per CTA, 129 x 5600 (175
# block columns) a shape its grid rule hands to variant 2
VARIANT_SHAPES = [(1, 32), (37, 64), (129, 5600), (257, 2240), (1000, 1152), (300, 12288), (4099, 1152)]
RING = (9,)


@pytest.mark.parametrize("M,d", VARIANT_SHAPES, ids=[f"{M}x{d}" for M, d in VARIANT_SHAPES])
def test_baseline_variants_bit_exact(cuda_device, M, d):
    """Register-prefetch and TMA-staged SQ/MX kernels agree bit for bit with the oracle
    (ragged final stage, odd block counts, a single block)."""
    x = synth.activation("pixart", M, d, seed=M * 7 + d)
    m = synth.sq_multipliers(x)
    xd, md = dev_bf16(x, cuda_device), dev_f32(m, cuda_device)
    rs, rm = oracle.sq_quantize(x, m), oracle.mx_quantize(x)
    for v in (1, 2):
        c, s = kq.sq_quantize_variant(v, xd, md)
        assert pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *rs)["ok"], ("sq", v)
        c, s = kq.mx_quantize_variant(v, xd)
        assert pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *rm)["ok"], ("mx", v)


@pytest.mark.parametrize("M,d", VARIANT_SHAPES, ids=[f"{M}x{d}" for M, d in VARIANT_SHAPES])
def test_kq_variants_sharing_arithmetic_are_identical(cuda_device, M, d):
    """Variants 2, 3 and 9 share the arithmetic, so their outputs are identical."""
    x = synth.activation("pixart", M, d, seed=M * 3 + d)
    F = synth.factors(d // 32, seed=d + 1)
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    c2, s2 = kq.kq_quantize_variant(2, xd, Fd)
    for v in (3,) + RING:
        cv, sv = kq.kq_quantize_variant(v, xd, Fd)
        assert bool((c2 == cv).all()) and bool((s2 == sv).all()), v
    F1 = synth.factors(1, seed=d, shared=True)
    c2, s2 = kq.kq_quantize_variant(2, xd, dev_f32(F1, cuda_device), shared=True)
    for v in (3,) + RING:
        cv, sv = kq.kq_quantize_variant(v, xd, dev_f32(F1, cuda_device), shared=True)
        assert bool((c2 == cv).all()) and bool((s2 == sv).all()), v
    # a column that falls back to the direct form (swap factor) alongside split ones
    F2 = F.copy()
    F2[0, 2] = np.array([[0, 1], [1, 0]], np.float32)
    c2, s2 = kq.kq_quantize_variant(2, xd, dev_f32(F2, cuda_device))
    for v in (3,) + RING:
        cv, sv = kq.kq_quantize_variant(v, xd, dev_f32(F2, cuda_device))
        assert bool((c2 == cv).all()) and bool((s2 == sv).all()), v


def test_bounded_wait_gives_up_and_context_stays_usable(cuda_device):
    """A staged CTA whose producer issues no copies: its waits run out, the
    device counter records it, and the next launches still work."""
    import torch

    kq.kq_wait_timeouts(reset=True)
    kq.kq_selftest_bounded_wait()
    torch.cuda.synchronize()
    assert kq.kq_wait_timeouts(reset=True) > 0
    M, d = 64, 128
    x = synth.activation("tiny", M, d, 0)
    xd = dev_bf16(x, cuda_device)
    c, s = kq.mx_quantize(xd)
    assert pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *oracle.mx_quantize(x))["ok"]
    # the staged kernels themselves (shared-memory opt-in, barrier set-up and
    # TMA ring of the kernel whose waits just ran out) still work
    c, s = kq.mx_quantize_variant(2, xd)
    assert pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *oracle.mx_quantize(x))["ok"]
    m = synth.sq_multipliers(x)
    c, s = kq.sq_quantize(xd, dev_f32(m, cuda_device))            # default: the staged kernel
    assert pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *oracle.sq_quantize(x, m))["ok"]
    torch.cuda.synchronize()
    assert kq.kq_wait_timeouts() == 0


def test_zero_rows_and_nondefault_stream(cuda_device):
    import torch

    M, d = 128, 4608
    x = synth.activation("pixart", M, d, 25)
    x[5] = 0
    F = synth.factors(d // 32, 25)
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    s = torch.cuda.Stream(device=cuda_device)
    with torch.cuda.stream(s):
        c, sc = kq.kq_quantize(xd, Fd)
    s.synchronize()
    c0, s0 = kq.kq_quantize(xd, Fd)
    assert bool((c == c0).all()) and bool((sc == s0).all())
    assert int(sc[5].max()) == 0 and int(c[5].max()) == 0


def test_empty_with_real_buffers(cuda_device):
    import torch

    x = torch.empty((0, 64), dtype=torch.bfloat16, device=cuda_device)
    c, s = kq.kq_quantize(x, torch.ones(2 * 20, device=cuda_device))
    assert c.shape == (0, 32) and s.shape == (0, 2)
    c, s = kq.mx_quantize(x)
    assert c.numel() == 0


def test_misaligned_pointer_is_rejected_and_context_stays_usable(cuda_device):
    import torch

    M, d = 4, 64
    base = torch.zeros(M * d + 8, dtype=torch.bfloat16, device=cuda_device)
    bad = base[1:1 + M * d].view(M, d)           # 2-byte offset
    with pytest.raises(kq.KroQuantError) as ei:
        kq.mx_quantize(bad)
    assert ei.value.status == kq.KQ_ERR_ALIGN
    good = base[8:8 + M * d].view(M, d)          # 16-byte offset
    c, s = kq.mx_quantize(good)
    torch.cuda.synchronize()
    assert int(s.max()) == 0


def test_extreme_magnitudes(cuda_device):
    M, d = 16, 64
    rng = np.random.default_rng(5)
    vals = rng.standard_normal((M, d)).astype(np.float32)
    vals[0] *= np.float32(2.0 ** 120)      # near the top of the range
    vals[1] *= np.float32(2.0 ** -128)     # subnormal bf16
    vals[2] = 0.0
    vals[3, ::2] = 0.0
    x = bf16(vals)
    I = np.tile(np.eye(2, dtype=np.float32), (d // 32, 5, 1, 1))
    c, s = kq.kq_quantize(dev_bf16(x, cuda_device), dev_f32(I, cuda_device))
    cr, sr = oracle.kq_quantize(x, I)
    np.testing.assert_array_equal(s.cpu().numpy(), sr)
    np.testing.assert_array_equal(c.cpu().numpy(), cr)
    # The plain MX path keeps the sign of a -0 input (bf16 underflow of tiny
    # negatives gives -0); the transform's sum turns it into +0, so MX is
    # compared with the oracle's MX, not with the identity-factor KQ result.
    c, s = kq.mx_quantize(dev_bf16(x, cuda_device))
    cm, sm = oracle.mx_quantize(x)
    np.testing.assert_array_equal(s.cpu().numpy(), sm)
    np.testing.assert_array_equal(c.cpu().numpy(), cm)


KQ_VARIANTS = (0, 1, 2, 3, 4) + RING


def test_unit_split_limits_near_the_top_of_the_range(cuda_device):
    """Factors at the limits of the unit-diagonal split (|b| = |c| = 16,
    diagonals 1/16) on inputs near 2^115: the split's intermediates U x grow
    by up to 17^5 and overflow fp32 there, while the transform itself (row
    sums of |K| = 1.0625^5) stays finite, so every variant must still match
    the oracle.  Column 1 has a factor beyond the split (|b| = 20) and runs
    the direct form."""
    M, d = 300, 128
    G = np.array([[1 / 16, 1.0], [1.0, 1 / 16]], np.float32)
    F = np.tile(G, (d // 32, 5, 1, 1))
    F[1, 2] = np.array([[1 / 20, 1.0], [1.0, 1 / 16]], np.float32)
    rng = np.random.default_rng(11)
    x = bf16(rng.standard_normal((M, d)).astype(np.float32) * np.float32(2.0 ** 115))
    cr, sr = oracle.kq_quantize(x, F)
    yr, ab = oracle.kq_transform(x, F, want_absbound=True)
    assert np.isfinite(yr).all() and int(sr.max()) < 0xFF
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    for v in KQ_VARIANTS:
        c, s = kq.kq_quantize_variant(v, xd, Fd)
        res = pc.check_kq(c.cpu().numpy(), s.cpu().numpy(), cr, sr, yr, ab)
        assert res["ok"], (v, res)
    # the fp32 transform export and the LU form take the same path
    y = kq.kq_transform_f32(xd, Fd).cpu().numpy()
    assert pc.check_transform(y, yr, ab)["bad"] == 0
    assert kq.kq_wait_timeouts() == 0


def test_transform_overflow_gives_the_nan_scale(cuda_device):
    """Where the transform of a finite block exceeds fp32 (here the unnormalised
    Hadamard factor [[1, 1], [1, -1]], row sums 2^5, on inputs near 2^126), the
    oracle writes the E8M0 NaN byte 0xFF and zero codes; so does every variant.
    Other blocks are unaffected."""
    M, d = 96, 256
    H = np.array([[1.0, 1.0], [1.0, -1.0]], np.float32)
    F = np.tile(H, (d // 32, 5, 1, 1))
    rng = np.random.default_rng(12)
    vals = rng.standard_normal((M, d)).astype(np.float32)
    vals[::3] *= np.float32(2.0 ** 126)          # every third row overflows
    x = bf16(vals)
    cr, sr = oracle.kq_quantize(x, F)
    assert (sr[::3] == 0xFF).all() and (cr[::3] == 0).all() and (sr[1::3] < 0xFF).all()
    xd, Fd = dev_bf16(x, cuda_device), dev_f32(F, cuda_device)
    for v in KQ_VARIANTS:
        c, s = kq.kq_quantize_variant(v, xd, Fd)
        c, s = c.cpu().numpy(), s.cpu().numpy()
        np.testing.assert_array_equal(s[::3], sr[::3], err_msg=f"variant {v}")
        np.testing.assert_array_equal(c[::3], cr[::3], err_msg=f"variant {v}")
        keep = np.ones(M, bool)
        keep[::3] = False
        yr, ab = oracle.kq_transform(x[keep], F, want_absbound=True)
        res = pc.check_kq(c[keep], s[keep], cr[keep], sr[keep], yr, ab)
        assert res["ok"], (v, res)
