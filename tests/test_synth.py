"""The seeded synthetic inputs (w4a4_mxfp4_post_b200.synth) keep the properties
the parity tests and the benchmark rely on: any row range can be regenerated
alone, the same seed gives the same bits, the recipe's structure is there."""
import ml_dtypes
import numpy as np
import pytest

from w4a4_mxfp4_post_b200 import synth


@pytest.mark.parametrize("model,M,d", [("pixart", 5000, 96), ("sana", 4500, 64), ("flux", 4608, 64),
                                       ("tiny", 64, 128)])
def test_row_ranges_equal_slices_of_the_full_matrix(model, M, d):
    full = synth.activation(model, M, d, 9)
    for r0, r1 in [(0, 1), (2047, 2049), (100, 4100), (M - 3, M), (M, M)]:
        if r1 > M:
            continue
        np.testing.assert_array_equal(synth.activation(model, M, d, 9, rows=(r0, r1)), full[r0:r1])


def test_same_seed_same_bits_other_seed_other_bits():
    a = synth.activation("pixart", 300, 128, 4)
    assert np.array_equal(a, synth.activation("pixart", 300, 128, 4))
    assert not np.array_equal(a, synth.activation("pixart", 300, 128, 5))


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.standard_normal(100000) * 3)).astype(np.float32)
    ref = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    np.testing.assert_array_equal(synth.bf16_bits_from_f32(x), ref)
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(ref), ref.view(ml_dtypes.bfloat16).astype(np.float32))


def test_outlier_channels_and_flux_text_rows():
    d = 1152
    x = synth.bf16_bits_to_f32(synth.activation("pixart", 4096, d, 1)).astype(np.float64)
    rms = np.sqrt((x * x).mean(axis=0))
    n_out = int(np.ceil(0.005 * d))
    top = np.argsort(rms)[-n_out:]
    assert np.median(rms[top]) > 10 * np.median(rms)            # the x50 outlier channels stand out
    M = 4608
    f = synth.bf16_bits_to_f32(synth.activation("flux", M, d, 3)).astype(np.float64)
    img, txt = f[: M - M // 9], f[M - M // 9:]
    k = int(np.ceil(0.01 * d))
    top_img = set(np.argsort(np.abs(img).max(axis=0))[-k:])
    top_txt = set(np.argsort(np.abs(txt).max(axis=0))[-k:])
    assert len(top_img & top_txt) < k // 2                      # text rows have their own outlier set


def test_factors_respect_the_determinant_floor():
    F = synth.factors(200, 7)
    det = F[:, :, 0, 0] * F[:, :, 1, 1] - F[:, :, 0, 1] * F[:, :, 1, 0]
    assert F.shape == (200, 5, 2, 2) and np.all(np.abs(det) >= 0.2)
    assert synth.factors(1, 7, shared=True).shape == (1, 5, 2, 2)


def test_mx_operand_ranges():
    c, s = synth.mx_operand(300, 640, 3)
    assert c.shape == (300, 320) and s.shape == (300, 20)
    assert c.dtype == np.uint8 and s.min() >= 112 and s.max() < 142
    assert len(np.unique(c)) == 256                             # every code byte occurs
