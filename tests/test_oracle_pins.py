"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against an independent source: numpy's and
scipy's library routines (np.kron, scipy.linalg.hadamard, np.linalg.inv/det),
ml_dtypes' FP4 E2M1 rounding, brute-force enumeration, closed forms, and the
hand-worked blocks of tests/golden/hand_blocks.txt.  They are chosen so that a
plausible slip in the oracle (factor order, transposed factor, dropped stage,
wrong scale offset, wrong tie rule, swapped nibbles, lost sign) fails at
least one of them.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg

import oracle
from conftest import GOLDEN, parse_blocks
from w4a4_mxfp4_post_b200 import synth

RNG = np.random.default_rng(12345)


def rand_factors(n, rng=RNG):
    return (np.eye(2) + 0.4 * rng.standard_normal((n, 5, 2, 2))).astype(np.float32)


def bf16(a):
    return synth.bf16_bits_from_f32(np.asarray(a, np.float32))


def f32(bits):
    return synth.bf16_bits_to_f32(bits)


# ---------------------------------------------------------------- Kronecker
def test_kron_expand_matches_numpy_kron():
    # KroQuant section 3.2, Eq. (4): K = G1 (x) G2 (x) G3 (x) G4 (x) G5.
    for F in rand_factors(20):
        ref = F[0].astype(np.float64)
        for k in range(1, 5):
            ref = np.kron(ref, F[k].astype(np.float64))
        np.testing.assert_allclose(oracle.kron_expand(F), ref, rtol=1e-15, atol=0)


def test_kron_hadamard_init_is_sylvester_hadamard():
    # Hadamard initialisation (Pith review, core discovery): identical factors
    # H2 give the Sylvester Hadamard matrix of order 32.
    H2 = np.array([[1, 1], [1, -1]], np.float32)
    K = oracle.kron_expand(np.stack([H2] * 5))
    np.testing.assert_array_equal(K, scipy.linalg.hadamard(32).astype(np.float64))
    # LU form of Eq. (6) with a = b = 1/sqrt(2), c = 1 is H2/sqrt(2): K K^T = I.
    a = b = 1 / np.sqrt(2.0)
    c = 1.0
    G = np.array([[1, 0], [c, 1]]) @ np.array([[a, b], [0, -1 / a]])
    np.testing.assert_allclose(G, H2 / np.sqrt(2.0), atol=1e-15)
    Kn = oracle.kron_expand(np.stack([G.astype(np.float32)] * 5))
    np.testing.assert_allclose(Kn @ Kn.T, np.eye(32), atol=1e-6)


def test_lu_factors_give_det_plus_one():
    # Eq. (6): G = L U with U = [[a, b], [0, -1/a]], L unit lower triangular, so
    # det G = -1; det(A (x) B) = det(A)^m det(B)^n makes det K = (-1)^80 = +1.
    rng = np.random.default_rng(7)
    for _ in range(10):
        F = []
        for _k in range(5):
            a, b, c = 0.5 + rng.random(), rng.standard_normal(), rng.standard_normal()
            F.append(np.array([[1, 0], [c, 1]]) @ np.array([[a, b], [0, -1 / a]]))
        F = np.array(F, np.float32)
        K = oracle.kron_expand(F)
        dets = np.prod([np.linalg.det(f.astype(np.float64)) for f in F]) ** 16
        assert np.linalg.det(K) == pytest.approx(dets, rel=1e-6)
        assert np.linalg.det(K) == pytest.approx(1.0, rel=1e-4)


def test_inverse_matches_kron_of_inverses():
    for F in rand_factors(10):
        K = oracle.kron_expand(F)
        Ki = oracle.inverse32(K)
        np.testing.assert_allclose(Ki @ K, np.eye(32), atol=1e-9)
        ref = np.linalg.inv(F[0].astype(np.float64))
        for k in range(1, 5):
            ref = np.kron(ref, np.linalg.inv(F[k].astype(np.float64)))
        np.testing.assert_allclose(Ki, ref, rtol=1e-9, atol=1e-12)


def tensor_apply(F, x):
    """(G1 (x) ... (x) G5) x as five 2x2 maps on the axes of x viewed as a 2x2x2x2x2 tensor."""
    t = x.astype(np.float64).reshape(-1, 2, 2, 2, 2, 2)
    for k in range(5):
        t = np.moveaxis(np.tensordot(F[k].astype(np.float64), t, axes=([1], [k + 1])), 0, k + 1)
    return t.reshape(x.shape)


def test_transform_matches_tensor_axis_form():
    # Independent formulation: a Kronecker product acts factor-by-factor on the
    # axes of the index tensor (axis 0 = most significant bit).
    M, d = 7, 96
    x = bf16(RNG.standard_normal((M, d)) * 3)
    F = rand_factors(d // 32)
    y, ab = oracle.kq_transform(x, F, want_absbound=True)
    xv = f32(x).reshape(M, d // 32, 32)
    ref = np.stack([tensor_apply(F[j], xv[:, j, :]) for j in range(d // 32)], axis=1).reshape(M, d)
    # y is the fp32 rounding of a double sum: within half an fp32 ulp (+ double noise).
    np.testing.assert_array_less(np.abs(y.astype(np.float64) - ref), np.abs(ref) * 2.0 ** -24 + 1e-12 * ab)
    # absbound is |K||x|
    absref = np.stack([tensor_apply(np.abs(F[j]), np.abs(xv[:, j, :])) for j in range(d // 32)],
                      axis=1).reshape(M, d)
    np.testing.assert_allclose(ab, absref, rtol=1e-13)


def test_transform_shared_equals_repeated_factors():
    M, d = 5, 160
    x = bf16(RNG.standard_normal((M, d)))
    F1 = rand_factors(1)
    y_sh = oracle.kq_transform(x, F1, shared=True)
    y_rep = oracle.kq_transform(x, np.repeat(F1, d // 32, axis=0))
    np.testing.assert_array_equal(y_sh, y_rep)


# ---------------------------------------------------------------- E2M1 / E8M0
def mld_codes(v):
    """E2M1 codes from ml_dtypes (RNE, saturating at 6, signed zero)."""
    return np.asarray(v, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_matches_ml_dtypes():
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    mids = (grid[1:] + grid[:-1]) / 2
    vals = [np.linspace(-7.99, 7.99, 20011), grid, -grid, mids, -mids,
            np.nextafter(mids, 0), np.nextafter(mids, 10), -np.nextafter(mids, 0), -np.nextafter(mids, 10),
            [6.5, 7.0, 7.9999, -7.0, 0.0, -0.0, 1e-30, -1e-30]]
    v = np.concatenate([np.asarray(a, np.float64) for a in vals]).astype(np.float32)
    ours = np.array([oracle.e2m1(float(t)) for t in v], np.uint8)
    np.testing.assert_array_equal(ours, mld_codes(v))


def test_e2m1_tie_table():
    # Ties go to the even code (OCP MX round-to-nearest-even).
    table = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6,
             -0.25: 8, -0.75: 10, -1.25: 10, -1.75: 12, -2.5: 12, -3.5: 14, -5.0: 14}
    for v, c in table.items():
        assert oracle.e2m1(v) == c, v


def e8m0_by_enumeration(amax):
    """The unique e with 2^(e+2) <= amax < 2^(e+3), clamped to [-127, 127]; 0 -> -127."""
    if amax == 0:
        return 0
    for e in range(-127 - 30, 128 + 1):
        if 2.0 ** (e + 2) <= amax < 2.0 ** (e + 3):
            return min(max(e, -127), 127) + 127
    raise AssertionError(amax)


def test_e8m0_bruteforce():
    rng = np.random.default_rng(3)
    vals = list(np.exp2(rng.uniform(-149, 128, 3000)).astype(np.float32))
    for k in range(-149, 128):
        p = np.float32(2.0 ** k)
        vals += [p, np.nextafter(p, np.float32(0)), np.nextafter(p, np.float32(np.inf))]
    vals += [np.float32(0.0), np.finfo(np.float32).max, np.finfo(np.float32).tiny]
    for a in vals:
        a = np.float32(a)
        if not np.isfinite(a):
            continue
        assert oracle.e8m0(float(a)) == e8m0_by_enumeration(float(a)), a
    assert oracle.e8m0(float("inf")) == 0xFF


def independent_mx(y):
    """MX block quantizer from enumeration (scale) and ml_dtypes (E2M1 rounding)."""
    y = np.asarray(y, np.float32).reshape(-1, 32)
    codes = np.zeros((y.shape[0], 16), np.uint8)
    scales = np.zeros(y.shape[0], np.uint8)
    for b in range(y.shape[0]):
        sb = e8m0_by_enumeration(float(np.max(np.abs(y[b]))))
        v = (y[b].astype(np.float64) * 2.0 ** (127 - sb)).astype(np.float32)
        c = mld_codes(v)
        codes[b] = c[0::2] | (c[1::2] << 4)
        scales[b] = sb
    return codes, scales


def test_mx_block_matches_independent_composition():
    rng = np.random.default_rng(11)
    for _ in range(300):
        y = (rng.standard_normal(32) * np.exp2(rng.integers(-120, 120))).astype(np.float32)
        if rng.random() < 0.3:
            y[rng.integers(32)] *= 40
        c, s = oracle.mx_block(y)
        ci, si = independent_mx(y)
        assert s == si[0]
        np.testing.assert_array_equal(c, ci[0])


def test_mx_quantize_matches_independent_composition():
    M, d = 33, 160
    x = synth.activation("pixart", M, d, seed=5)
    codes, scales = oracle.mx_quantize(x)
    ci, si = independent_mx(f32(x).reshape(-1, 32))
    np.testing.assert_array_equal(codes.reshape(-1, 16), ci)
    np.testing.assert_array_equal(scales.reshape(-1), si)


def test_power_of_two_invariance():
    # Scaling x by 2^k adds k to every scale byte and leaves the codes unchanged
    # (away from the clamps): the MX scale is a power of two.
    x = synth.activation("tiny", 16, 128, seed=3)
    F = rand_factors(4)
    c0, s0 = oracle.kq_quantize(x, F)
    for k in (-20, -3, 1, 7, 30):
        xk = bf16(f32(x) * np.float32(2.0 ** k))
        ck, sk = oracle.kq_quantize(xk, F)
        np.testing.assert_array_equal(ck, c0)
        np.testing.assert_array_equal(sk.astype(int), s0.astype(int) + k)


# ---------------------------------------------------------------- cross-identities
def test_identity_factors_equal_mx():
    x = synth.activation("pixart", 17, 192, seed=9)
    I = np.tile(np.eye(2, dtype=np.float32), (6, 5, 1, 1))
    np.testing.assert_array_equal(oracle.kq_quantize(x, I)[0], oracle.mx_quantize(x)[0])
    np.testing.assert_array_equal(oracle.kq_quantize(x, I)[1], oracle.mx_quantize(x)[1])


def test_sq_unit_multiplier_equals_mx_and_matches_numpy_product():
    x = synth.activation("pixart", 19, 256, seed=10)
    one = np.ones(256, np.float32)
    np.testing.assert_array_equal(oracle.sq_quantize(x, one)[0], oracle.mx_quantize(x)[0])
    m = synth.sq_multipliers(x)
    prod = f32(x) * m[None, :]          # numpy fp32 multiply: one correctly rounded product
    ci, si = independent_mx(prod.reshape(-1, 32))
    c, s = oracle.sq_quantize(x, m)
    np.testing.assert_array_equal(c.reshape(-1, 16), ci)
    np.testing.assert_array_equal(s.reshape(-1), si)


def test_kq_quantize_is_transform_then_mx():
    x = synth.activation("pixart", 9, 128, seed=12)
    F = rand_factors(4)
    y = oracle.kq_transform(x, F)
    ci, si = independent_mx(y.reshape(-1, 32))
    c, s = oracle.kq_quantize(x, F)
    np.testing.assert_array_equal(c.reshape(-1, 16), ci)
    np.testing.assert_array_equal(s.reshape(-1), si)


def test_diagonal_power_of_two_factors_scale_channels():
    # diag(2^a, 2^b) factors multiply channel i by 2^(sum of chosen exponents):
    # kq equals mx of the channel-scaled input.
    x = synth.activation("pixart", 8, 64, seed=13)
    ex = np.array([[1, -2], [0, 3], [2, 0], [-1, 1], [0, 0]])
    F = np.stack([np.diag(2.0 ** e).astype(np.float32) for e in ex])
    scale = np.ones(32)
    for i in range(32):
        scale[i] = 2.0 ** sum(ex[k][(i >> (4 - k)) & 1] for k in range(5))
    xs = bf16(f32(x) * np.tile(scale, 2)[None, :].astype(np.float32))
    np.testing.assert_array_equal(oracle.kq_quantize(x, np.stack([F, F]))[0], oracle.mx_quantize(xs)[0])


# ---------------------------------------------------------------- fold
def test_fold_gives_exact_product_identity():
    # X W^T == (X T^T)(W T^-1)^T, the invertibility the fold relies on.
    M, N, d = 12, 10, 128
    x = synth.activation("tiny", M, d, seed=0)
    W = synth.weights(N, d, seed=0)
    F = synth.factors(d // 32, seed=0)
    Wf, abw = oracle.fold_weights(W, F, want_absbound=True)
    xv = f32(x).astype(np.float64).reshape(M, d // 32, 32)
    Y = np.stack([tensor_apply(F[j], xv[:, j, :]) for j in range(d // 32)], axis=1).reshape(M, d)
    lhs = f32(x).astype(np.float64) @ W.astype(np.float64).T
    rhs = Y @ Wf.astype(np.float64).T
    bound = (np.abs(Y) @ abw.T) * 2.0 ** -23 + 1e-12
    np.testing.assert_array_less(np.abs(lhs - rhs), bound)
    # and the folded weights are W times the library inverse of every K^(j)
    Kinv = [np.linalg.inv(oracle.kron_expand(F[j])) for j in range(d // 32)]
    ref = np.concatenate([W[:, 32 * j:32 * j + 32].astype(np.float64) @ Kinv[j] for j in range(d // 32)], axis=1)
    np.testing.assert_array_less(np.abs(Wf - ref), abw * 2.0 ** -23 + 1e-30)


# ---------------------------------------------------------------- hand-worked
@pytest.mark.parametrize("case", parse_blocks(os.path.join(GOLDEN, "hand_blocks.txt")), ids=lambda c: c["name"])
def test_hand_worked_blocks(case):
    x = bf16(case["x"])
    codes, scales = oracle.kq_quantize(x, case["factors"])
    assert scales[0, 0] == case["scale"]
    np.testing.assert_array_equal(codes[0], case["codes"])


def test_hand_worked_fixture_inputs_are_bf16_exact():
    for case in parse_blocks(os.path.join(GOLDEN, "hand_blocks.txt")):
        if case["name"] in ("ties_and_saturation", "negative_ties"):
            continue  # these carry a deliberate non-exact +-0.1
        np.testing.assert_array_equal(f32(bf16(case["x"])), case["x"])


# ---------------------------------------------------------------- LU form (Eq. 6) and FWHT baseline
def lu_np(a, b, c):
    return np.array([[1, 0], [c, 1]], np.float64) @ np.array([[a, b], [0, -1 / a]], np.float64)


def rand_lu(n, rng):
    P = np.empty((n, 5, 3), np.float32)
    P[..., 0] = (0.6 + 0.8 * rng.random((n, 5))) * rng.choice([-1, 1], (n, 5))
    P[..., 1] = 0.4 * rng.standard_normal((n, 5))
    P[..., 2] = 0.4 * rng.standard_normal((n, 5))
    return P


def test_lu_expansion_matches_numpy_kron_of_lu_products():
    rng = np.random.default_rng(21)
    for P in rand_lu(10, rng):
        ref = lu_np(*map(float, P[0]))
        for k in range(1, 5):
            ref = np.kron(ref, lu_np(*map(float, P[k])))
        np.testing.assert_allclose(oracle.kron_expand_lu(P), ref, rtol=1e-13, atol=1e-15)
        assert np.linalg.det(oracle.kron_expand_lu(P)) == pytest.approx(1.0, rel=1e-8)


def test_lu_hadamard_initialisation():
    a = np.float32(1 / np.sqrt(2.0))
    P = np.tile(np.array([a, a, 1.0], np.float32), (5, 1))
    K = oracle.kron_expand_lu(P)
    np.testing.assert_allclose(K, scipy.linalg.hadamard(32) / np.sqrt(32.0), atol=3e-7)


def test_lu_transform_agrees_with_factor_form():
    rng = np.random.default_rng(22)
    M, d = 9, 128
    x = synth.activation("pixart", M, d, 22)
    P = rand_lu(d // 32, rng)
    F = np.array([[lu_np(*map(float, P[j, k])) for k in range(5)] for j in range(d // 32)]).astype(np.float32)
    y_lu, ab = oracle.kq_transform_lu(x, P, want_absbound=True)
    y_f = oracle.kq_transform(x, F)
    # the factor form rounds G to fp32 first: a few fp32 ulps of |K||x|
    np.testing.assert_array_less(np.abs(y_lu.astype(np.float64) - y_f), 1e-6 * ab + 1e-30)
    c, s = oracle.kq_quantize_lu(x, P)
    ci, si = independent_mx(y_lu.reshape(-1, 32))
    np.testing.assert_array_equal(c.reshape(-1, 16), ci)
    np.testing.assert_array_equal(s.reshape(-1), si)


@pytest.mark.parametrize("H", [32, 64, 128, 256])
def test_fwht_matches_scipy_hadamard(H):
    M, d = 5, 512
    x = synth.activation("pixart", M, d, H)
    y, ab = oracle.fwht_transform(x, H, want_absbound=True)
    xv = f32(x).astype(np.float64).reshape(M, d // H, H)
    ref = (xv @ scipy.linalg.hadamard(H).T.astype(np.float64) / np.sqrt(H)).reshape(M, d)
    np.testing.assert_array_less(np.abs(y - ref), np.abs(ref) * 2.0 ** -24 + 1e-12 * ab + 1e-30)
    # orthonormal: energy is preserved block by block (Parseval)
    np.testing.assert_allclose((ref ** 2).reshape(M, -1, H).sum(-1), (xv ** 2).sum(-1), rtol=1e-12)
    np.testing.assert_allclose(ab, np.repeat(np.abs(xv).sum(-1), H, axis=1).reshape(M, d) / np.sqrt(H), rtol=1e-13)
    c, s = oracle.fwht_quantize(x, H)
    ci, si = independent_mx(y.reshape(-1, 32))
    np.testing.assert_array_equal(c.reshape(-1, 16), ci)
    np.testing.assert_array_equal(s.reshape(-1), si)


def test_fwht_32_is_kroquant_with_hadamard_factors():
    M, d = 7, 96
    x = synth.activation("pixart", M, d, 23)
    F = np.tile(np.array([[1, 1], [1, -1]], np.float32) / np.float32(np.sqrt(2.0)), (d // 32, 5, 1, 1))
    y_h, ab = oracle.fwht_transform(x, 32, want_absbound=True)
    y_k = oracle.kq_transform(x, F)
    np.testing.assert_array_less(np.abs(y_h.astype(np.float64) - y_k), 1e-6 * ab + 1e-30)


# ---------------------------------------------------------------- decode and inverse
def test_dequantize_matches_ml_dtypes_decode():
    rng = np.random.default_rng(31)
    M, d = 6, 128
    codes = rng.integers(0, 256, (M, d // 2), dtype=np.uint8)
    scales = rng.integers(0, 255, (M, d // 32), dtype=np.uint8)     # 0..254: finite
    out = oracle.mx_dequantize(codes, scales)
    nib = np.empty((M, d), np.uint8)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    vals = nib.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    np.testing.assert_array_equal(out, (vals * np.repeat(sc, 32, axis=1)).astype(np.float32))
    s255 = scales.copy()
    s255[0, 0] = 0xFF
    assert np.isnan(oracle.mx_dequantize(codes, s255)[0, :32]).all()


def test_round_trip_error_is_within_half_a_step():
    # MX round trip: |x - x^| <= half the E2M1 spacing at |x| (times 2^e), except
    # where |x| 2^-e is beyond the largest grid point 6 (saturation).
    x = synth.activation("pixart", 64, 256, 33)
    c, s = oracle.mx_quantize(x)
    xh = oracle.mx_dequantize(c, s).astype(np.float64)
    xv = f32(x).astype(np.float64)
    e = np.repeat(s.astype(np.int64) - 127, 32, axis=1)
    a = np.abs(xv) * 2.0 ** -e
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    assert np.all(a <= 8)
    ok = np.abs(xv - xh) * 2.0 ** -e <= np.where(a > 6, a - 6, step / 2) + 1e-12
    assert ok.all()


def test_inverse_undoes_the_transform():
    M, d = 8, 128
    x = synth.activation("pixart", M, d, 34)
    F = rand_factors(d // 32)
    y = oracle.kq_transform(x, F)
    xr, ab = oracle.kq_inverse(y, F, want_absbound=True)
    np.testing.assert_array_less(np.abs(xr.astype(np.float64) - f32(x)), 1e-5 * ab + 1e-30)
    # and equals the library inverse of each dense block
    Kinv = [np.linalg.inv(oracle.kron_expand(F[j])) for j in range(d // 32)]
    ref = np.concatenate([y[:, 32 * j:32 * j + 32].astype(np.float64) @ Kinv[j].T for j in range(d // 32)], axis=1)
    np.testing.assert_array_less(np.abs(xr - ref), ab * 2.0 ** -23 + 1e-30)


# ---------------------------------------------------------------- fused normalisation (producer) + quantizer
def test_norm_kq_matches_torch_layer_norm_then_kron():
    import torch

    M, d, ns, eps = 12, 128, 3, 1e-6
    h = synth.activation("pixart", M, d, 51)
    rng = np.random.default_rng(51)
    gamma = (0.2 * rng.standard_normal((ns, d))).astype(np.float32)
    beta = (0.1 * rng.standard_normal((ns, d))).astype(np.float32)
    F = rand_factors(d // 32)
    out = oracle.norm_kq(h, gamma, beta, eps, F, want=("codes", "y", "absb"))
    hv = torch.from_numpy(f32(h).astype(np.float64))
    ln = torch.nn.functional.layer_norm(hv, (d,), eps=eps).numpy()          # library LayerNorm
    g64 = np.repeat(gamma.astype(np.float64), M // ns, axis=0)
    b64 = np.repeat(beta.astype(np.float64), M // ns, axis=0)
    xm = ln * (1 + g64) + b64
    ref = np.stack([tensor_apply(F[j], xm[:, 32 * j:32 * j + 32]) for j in range(d // 32)], 1).reshape(M, d)
    np.testing.assert_array_less(np.abs(out["y"] - ref), np.abs(ref) * 2.0 ** -24 + 1e-9 * out["absb"] + 1e-30)
    ci, si = independent_mx(out["y"].reshape(-1, 32))
    np.testing.assert_array_equal(out["codes"].reshape(-1, 16), ci)
    np.testing.assert_array_equal(out["scales"].reshape(-1), si)
