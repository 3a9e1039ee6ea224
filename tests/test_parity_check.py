"""The agreement checker itself, on oracle outputs with planted differences (CPU only)."""
import numpy as np

import oracle
import parity_check as pc
from w4a4_mxfp4_post_b200 import synth


def data():
    M, d = 40, 128
    x = synth.activation("pixart", M, d, 31)
    F = synth.factors(d // 32, 31)
    c, s = oracle.kq_quantize(x, F)
    y, ab = oracle.kq_transform(x, F, want_absbound=True)
    return c, s, y, ab


def test_identical_outputs_pass():
    c, s, y, ab = data()
    r = pc.check_kq(c, s, c, s, y, ab)
    assert r["ok"] and r["code_mismatch"] == 0


def test_planted_code_flip_fails():
    c, s, y, ab = data()
    bad = c.copy()
    # flip the magnitude of a code whose value is far from every boundary
    v = np.abs(np.ldexp(y.astype(np.float64), -(s.astype(np.int64).repeat(32, axis=1) - 127)))
    far = np.abs(v[:, :, None] - pc.BOUNDARIES[None, None, :]).min(axis=2) > 0.1
    r_, i_ = np.argwhere(far)[0]
    bad[r_, i_ // 2] ^= (1 << (4 * (i_ % 2)))
    r = pc.check_kq(bad, s, c, s, y, ab)
    assert not r["ok"] and r["code_mismatch_nonexempt"] == 1


def test_planted_scale_change_fails():
    c, s, y, ab = data()
    bad = s.copy()
    bad[3, 1] += 1
    r = pc.check_kq(c, bad, c, s, y, ab)
    assert not r["ok"] and r["scale_mismatch_unflagged"] == 1


def test_near_boundary_flip_is_exempt():
    # a value placed on a rounding boundary: either neighbouring code is accepted
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 6.0          # amax 6 -> e = 0
    x[0, 1] = 2.5          # tie between codes 4 (2.0) and 5 (3.0)
    xb = synth.bf16_bits_from_f32(x)
    F = np.tile(np.eye(2, dtype=np.float32), (1, 5, 1, 1))
    c, s = oracle.kq_quantize(xb, F)
    y, ab = oracle.kq_transform(xb, F, want_absbound=True)
    other = c.copy()
    other[0, 0] = (other[0, 0] & 0x0F) | (5 << 4)
    r = pc.check_kq(other, s, c, s, y, ab)
    assert r["ok"] and r["code_mismatch_exempt"] == 1


def test_exact_checker():
    c, s, y, ab = data()
    assert pc.check_exact(c, s, c, s)["ok"]
    bad = c.copy()
    bad[0, 0] ^= 0x80
    assert not pc.check_exact(bad, s, c, s)["ok"]


def test_transform_check():
    c, s, y, ab = data()
    assert pc.check_transform(y, y, ab)["bad"] == 0
    y2 = y.copy()
    y2[1, 5] += np.float32(3e-5) * np.float32(ab[1, 5])
    assert pc.check_transform(y2, y, ab)["bad"] == 1
