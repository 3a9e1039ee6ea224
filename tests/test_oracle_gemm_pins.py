"""Pins of the oracle's W4A4 pieces: the scale-factor layout, the fp32-input
MXFP4 quantizer and the MXFP4 x MXFP4 product.

The product is pinned by hand-worked cases (tests/golden/hand_gemm.txt), by a
float64 numpy matmul of the decoded operands (the decode itself is pinned
against ml_dtypes in test_oracle_pins.py), and by the transpose identity.  The
scale-factor layout is pinned by offsets worked out by hand from the stated
layout of the tensor core's scale operand and by being a bijection.
"""
import os

import numpy as np
import pytest

import oracle
from conftest import GOLDEN

RNG = np.random.default_rng(1234)


def parse_gemm(path):
    cases, cur = [], None
    with open(path) as fh:
        for raw in fh:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            val = val.strip()
            if key == "case":
                cur = {"name": val}
                cases.append(cur)
            elif key == "shape":
                cur["shape"] = tuple(int(t) for t in val.split())
            elif key in ("a_codes", "a_scales", "b_codes", "b_scales"):
                rows = [[int(t, 16) for t in r.split()] for r in val.split("|")]
                cur[key] = np.array(rows, np.uint8)
            elif key == "d":
                cur["d"] = np.array([float(t) for t in val.split()], np.float64)
            else:
                raise ValueError(f"bad golden line: {raw!r}")
    return cases


GEMM_CASES = parse_gemm(os.path.join(GOLDEN, "hand_gemm.txt"))


@pytest.mark.parametrize("case", GEMM_CASES, ids=[c["name"] for c in GEMM_CASES])
def test_hand_worked_gemm(case):
    M, N, K = case["shape"]
    assert case["a_codes"].shape == (M, K // 2) and case["b_codes"].shape == (N, K // 2)
    D = oracle.mxf4_gemm(case["a_codes"], case["a_scales"], case["b_codes"], case["b_scales"])
    np.testing.assert_array_equal(D.ravel(), case["d"])


def rand_mx(rows, K, rng):
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(100, 150, (rows, K // 32), dtype=np.uint8)
    return codes, scales


@pytest.mark.parametrize("M,N,K", [(3, 5, 32), (17, 9, 160), (40, 33, 512)])
def test_gemm_is_matmul_of_decoded_operands(M, N, K):
    ca, sa = rand_mx(M, K, RNG)
    cb, sb = rand_mx(N, K, RNG)
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    A = oracle.mx_dequantize(ca, sa).astype(np.float64)
    B = oracle.mx_dequantize(cb, sb).astype(np.float64)
    ref = A @ B.T
    # both sides are exact products summed in double: differences are double rounding only
    assert np.all(np.abs(D - ref) <= 1e-12 * np.abs(A) @ np.abs(B).T)
    np.testing.assert_allclose(absd, np.abs(A) @ np.abs(B).T, rtol=1e-12)


def test_gemm_transpose_identity_and_row_sampling():
    ca, sa = rand_mx(12, 96, RNG)
    cb, sb = rand_mx(7, 96, RNG)
    D = oracle.mxf4_gemm(ca, sa, cb, sb)
    Dt = oracle.mxf4_gemm(cb, sb, ca, sa)
    np.testing.assert_array_equal(D, Dt.T)
    rows = np.array([11, 0, 5])
    np.testing.assert_array_equal(oracle.mxf4_gemm(ca, sa, cb, sb, rows=rows), D[rows])


def test_sf_offsets_worked_by_hand():
    # 32 lanes x 16 bytes per 512-byte unit; lane l holds rows l, l+32, l+64,
    # l+96 at byte 4*(row group) + block; units ordered row-group major.
    nb = 8                                    # two units per 128-row group
    assert oracle.sf_offset(0, 0, nb) == 0
    assert oracle.sf_offset(1, 0, nb) == 16
    assert oracle.sf_offset(31, 0, nb) == 496
    assert oracle.sf_offset(32, 0, nb) == 4
    assert oracle.sf_offset(64, 0, nb) == 8
    assert oracle.sf_offset(96, 0, nb) == 12
    assert oracle.sf_offset(0, 3, nb) == 3
    assert oracle.sf_offset(0, 4, nb) == 512
    assert oracle.sf_offset(127, 7, nb) == 512 + 31 * 16 + 3 * 4 + 3
    assert oracle.sf_offset(128, 0, nb) == 1024
    assert oracle.sf_offset(128, 0, 70) == 18 * 512          # ceil(70 / 4) = 18 units per group
    assert oracle.sf_bytes(300, 70) == 3 * 18 * 512
    assert oracle.sf_bytes(128, 4) == 512


@pytest.mark.parametrize("rows,nb", [(1, 1), (128, 4), (300, 70), (257, 9)])
def test_sf_layout_is_a_bijection_onto_the_buffer(rows, nb):
    R = -(-rows // 128) * 128
    C = -(-nb // 4) * 4
    offs = np.array([oracle.sf_offset(r, j, nb) for r in range(R) for j in range(C)])
    assert offs.min() == 0 and offs.max() == oracle.sf_bytes(rows, nb) - 1
    assert np.unique(offs).size == offs.size == oracle.sf_bytes(rows, nb)


def test_scales_to_sf_places_every_scale_and_the_odd_pad():
    rows, nb = 200, 7
    sc = RNG.integers(0, 255, (rows, nb), dtype=np.uint8)
    sf = oracle.scales_to_sf(sc)
    back = np.array([[sf[oracle.sf_offset(r, j, nb)] for j in range(nb)] for r in range(rows)], np.uint8)
    np.testing.assert_array_equal(back, sc)
    pads = np.array([sf[oracle.sf_offset(r, nb, nb)] for r in range(rows)])
    assert np.all(pads == 0)
    mask = oracle.sf_defined_mask(rows, nb)
    assert mask.sum() == rows * (nb + 1)
    assert np.all(sf[~mask] == 0xFF)


def test_mx_quantize_f32_equals_bf16_path_on_bf16_values():
    import ml_dtypes

    x = (RNG.standard_normal((33, 96)) * np.exp(RNG.standard_normal((1, 96)))).astype(np.float32)
    xb = x.astype(ml_dtypes.bfloat16)
    c1, s1 = oracle.mx_quantize_f32(xb.astype(np.float32))
    c2, s2 = oracle.mx_quantize(xb.view(np.uint16))
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)


def test_mx_quantize_f32_round_trip_error_bound():
    x = (RNG.standard_normal((16, 128)) * 3).astype(np.float32)
    c, s = oracle.mx_quantize_f32(x)
    xr = oracle.mx_dequantize(c, s).astype(np.float64)
    # per block with scale 2^e: scaled values lie in [0, 8); below 6 the E2M1
    # grid step is at most 2, so rounding moves a value by at most 1 * 2^e;
    # values in (6, 8) saturate to 6, moving by less than 2 * 2^e
    e = np.repeat(s.astype(np.int64) - 127, 32, axis=1)
    v = np.abs(x) / np.ldexp(1.0, e)
    bound = np.where(v <= 6, 1.0, 2.0) * np.ldexp(1.0, e)
    assert np.all(np.abs(xr - x) <= bound)
    assert np.any(v > 6)            # the saturating branch is exercised


def test_w4a4_chain_computes_x_wt_on_the_oracle():
    """The chain the W4A4 consumer implements, on the oracle alone: with
    Hadamard factors, (MXFP4(X T^T)) (MXFP4(W T^-1))^T approximates X W^T
    better than plain MXFP4 on both operands, and dropping the fold (W left
    untransformed) destroys it.  Pins that the fold pairs with the transform
    (T^-1, not T or T^T) and that the product contracts the right indices."""
    from w4a4_mxfp4_post_b200 import synth

    M, N, d = 128, 96, 256
    x = synth.activation("pixart", M, d, 3)
    W = synth.weights(N, d, 3)
    s = np.float32(1.0 / np.sqrt(2.0))
    H = np.tile(np.array([[s, s], [s, -s]], np.float32), (d // 32, 5, 1, 1))
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ W.astype(np.float64).T
    ca, sa = oracle.kq_quantize(x, H)

    def rel(D):
        return np.linalg.norm(D - ref) / np.linalg.norm(ref)

    cb, sb = oracle.mx_quantize_f32(oracle.fold_weights(W, H))
    folded = rel(oracle.mxf4_gemm(ca, sa, cb, sb))
    cbu, sbu = oracle.mx_quantize_f32(W)
    unfolded = rel(oracle.mxf4_gemm(ca, sa, cbu, sbu))
    cam, sam = oracle.mx_quantize(x)
    plain = rel(oracle.mxf4_gemm(cam, sam, cbu, sbu))
    assert folded < plain < 0.5, (folded, plain)
    assert unfolded > 0.9, unfolded
