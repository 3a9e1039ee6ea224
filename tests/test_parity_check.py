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
    r = pc.check_kq(c, s, c, s, y, ab, pool=False)
    assert r["ok"] and r["code_mismatch"] == 0


def test_planted_code_flip_fails():
    c, s, y, ab = data()
    bad = c.copy()
    # flip the magnitude of a code whose value is far from every boundary
    v = np.abs(np.ldexp(y.astype(np.float64), -(s.astype(np.int64).repeat(32, axis=1) - 127)))
    far = np.abs(v[:, :, None] - pc.BOUNDARIES[None, None, :]).min(axis=2) > 0.1
    r_, i_ = np.argwhere(far)[0]
    bad[r_, i_ // 2] ^= (1 << (4 * (i_ % 2)))
    r = pc.check_kq(bad, s, c, s, y, ab, pool=False)
    assert not r["ok"] and r["code_mismatch_nonexempt"] == 1


def test_planted_scale_change_fails():
    c, s, y, ab = data()
    bad = s.copy()
    bad[3, 1] += 1
    r = pc.check_kq(c, bad, c, s, y, ab, pool=False)
    assert not r["ok"] and r["scale_mismatch_unflagged"] == 1 and r["scale_mismatch"] == 1


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
    r = pc.check_kq(other, s, c, s, y, ab, pool=False)
    assert r["ok"] and r["code_mismatch_exempt"] == 1
    # exactly on the boundary: inside the boundary-relative window too
    assert r["code_mismatch_exempt_outside_rel"] == 0


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


def test_flagged_scale_mismatch_counts_against_the_pooled_rate():
    # amax exactly 4 = 2^2: the block is flagged (a tolerance-sized error could
    # take either exponent); its mismatch passes the case but enters the pool
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 4.0
    xb = synth.bf16_bits_from_f32(x)
    F = np.tile(np.eye(2, dtype=np.float32), (1, 5, 1, 1))
    c, s = oracle.kq_quantize(xb, F)
    y, ab = oracle.kq_transform(xb, F, want_absbound=True)
    bad = s.copy()
    bad[0, 0] -= 1
    r = pc.check_kq(c, bad, c, s, y, ab, pool=False)
    # allowed per case, counted against the pooled rate
    assert r["flagged_blocks"] == 1 and r["scale_mismatch_flagged"] == 1 and r["ok"]
    assert not pc.pooled_verdict({"cases": 1, "codes": 32, "blocks": 1, "code_mismatch_exempt": 0,
                                  "code_mismatch_exempt_outside_rel": 0, "flagged_blocks": 1,
                                  "scale_mismatch_flagged": 1})["ok"]


def test_sign_of_zero_flip_is_exempt_but_outside_the_relative_window():
    # y_1 = x_0 - x_1 cancels exactly under the factor [[1, 1], [1, -1]] on
    # the lowest index bit: the oracle codes +0; a -0 (0x8) is within the
    # |K||x| window of the zero boundary but not within 1e-5 of a boundary b > 0
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 3.0
    x[0, 1] = 3.0
    xb = synth.bf16_bits_from_f32(x)
    F = np.tile(np.eye(2, dtype=np.float32), (1, 5, 1, 1))
    F[0, 4] = np.array([[1.0, 1.0], [1.0, -1.0]], np.float32)
    c, s = oracle.kq_quantize(xb, F)
    y, ab = oracle.kq_transform(xb, F, want_absbound=True)
    assert y[0, 1] == 0.0 and (c[0, 0] >> 4) == 0
    other = c.copy()
    other[0, 0] |= 0x80
    r = pc.check_kq(other, s, c, s, y, ab, pool=False)
    assert r["ok"] and r["code_mismatch_exempt"] == 1 and r["code_mismatch_exempt_outside_rel"] == 1


def test_pooled_rate():
    # one exempt mismatch per 1e6 codes passes, more fails; the rate is over
    # every code of every pooled case
    ok = pc.pooled_verdict({"cases": 2, "codes": 2_000_000, "blocks": 62_500, "code_mismatch_exempt": 2,
                            "code_mismatch_exempt_outside_rel": 0, "flagged_blocks": 0})
    assert ok["ok"] and ok["exempt_rate"] == 1e-6
    bad = pc.pooled_verdict({"cases": 2, "codes": 2_000_000, "blocks": 62_500, "code_mismatch_exempt": 3,
                             "code_mismatch_exempt_outside_rel": 0, "flagged_blocks": 0})
    assert not bad["ok"]


def test_unpooled_checks_leave_the_pool_alone():
    before = dict(pc.POOL)
    c, s, y, ab = data()
    pc.check_kq(c, s, c, s, y, ab, pool=False)
    assert pc.POOL == before


def test_gemm_check_rms_statistic_catches_a_dropped_k_block():
    # exact product rounded to fp32: passes both criteria
    K = 1152
    ca, sa = synth.mx_operand(64, K, 5)
    cb, sb = synth.mx_operand(48, K, 6)
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    ok = pc.check_gemm(D.astype(np.float32), D, absd, K, False)
    assert ok["ok"] and ok["rms_rel"] < ok["rms_bound"] / 10
    # the last 64-element K step left out of every output: the statistic,
    # taken over all outputs, is far above its bound
    ca2 = ca.copy()
    ca2[:, -32:] = 0
    r = pc.check_gemm(oracle.mxf4_gemm(ca2, sa, cb, sb), D, absd, K, False)
    assert not r["ok"] and r["rms_rel"] > 100 * r["rms_bound"]
    # an error of a few hundred fp32 roundings per output, everywhere: within
    # the worst-case K * 2^-23 bound but not the sqrt(K) statistic
    noisy = D + 300 * 2.0 ** -24 * absd * np.where(np.arange(D.size).reshape(D.shape) % 2, 1, -1)
    r2 = pc.check_gemm(noisy, D, absd, K, False)
    assert r2["bad"] == 0 and not r2["ok"]
