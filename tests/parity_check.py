"""Agreement criteria between the CUDA path and the CPU oracle.

KroQuant quantizer (transform + MXFP4), with y_ref the oracle's fp32 transform
and ab = |K||x| (the scale of a dot product's rounding error):

  transform  |y_gpu - y_ref| <= 1e-5 * ab                    (relative error
             taken against |K||x|, the standard dot-product error scale; a
             per-element relative test is ill-posed where y ~ 0)
  scales     bit-exact, except in "flagged" blocks, whose oracle amax lies
             within the transform tolerance of a power of two (a legitimate
             fp32 evaluation may then take the neighbouring exponent); flagged
             mismatches are counted and their codes left out of the code check
  codes      bit-exact, except where the oracle's scaled value v = y_ref 2^-e
             lies within w = 1e-5 * ab * 2^-e of a rounding boundary of E2M1
             (+-0.25, +-0.75, ..., +-5, or 0 for the sign of a zero); such
             "exempt" mismatches are counted and must stay <= 1e-6 of all codes;
             any other mismatch fails.  (The 1e-6 rate is rounded up to a
             whole code, so a case of fewer than 1e6 codes may show one.)

SmoothQuant and plain MXFP4: codes and scales bit-exact, no exemptions (the
fp32 product x * m is correctly rounded on both sides).
"""
from __future__ import annotations

import math

import numpy as np

BOUNDARIES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
REL = 1e-5
EXEMPT_FRACTION = 1e-6


def nibbles(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def allowed(n: int) -> int:
    """Exempt mismatches allowed among n results: 1e-6 of them, rounded up to a whole one.

    The rate bound is statistical; below a million codes a floor would allow
    none, although one near-boundary flip is then expected now and then.
    """
    return math.ceil(EXEMPT_FRACTION * n)


def scale_band_flags(y_ref: np.ndarray, ab: np.ndarray) -> np.ndarray:
    """[nblocks] True where the block amax can legitimately cross a power of two."""
    yb = np.abs(y_ref.reshape(-1, 32)).astype(np.float64)
    amax = yb.max(axis=1)
    tol = REL * ab.reshape(-1, 32).max(axis=1)
    lo = np.maximum(amax - tol, 0.0)
    hi = amax + tol
    _, elo = np.frexp(lo)
    _, ehi = np.frexp(hi)
    return (elo != ehi) & (hi > 0)


def check_transform(y_gpu, y_ref, ab):
    err = np.abs(y_gpu.astype(np.float64) - y_ref.astype(np.float64))
    bound = REL * ab + 1e-37
    bad = int(np.count_nonzero(err > bound))
    worst = float(np.max(err / (ab + 1e-37))) if err.size else 0.0
    return {"bad": bad, "worst_rel_to_absbound": worst}


def check_kq(codes_gpu, scales_gpu, codes_ref, scales_ref, y_ref, ab):
    """Counts per the criteria above; `ok` is the verdict."""
    sg = np.asarray(scales_gpu).reshape(-1)
    sr = np.asarray(scales_ref).reshape(-1)
    nblk = sr.size
    flagged = scale_band_flags(y_ref, ab)
    smis = sg != sr
    scale_bad = int(np.count_nonzero(smis & ~flagged))
    scale_flagged_mis = int(np.count_nonzero(smis & flagged))
    keep = ~smis                                   # blocks whose codes are compared
    cg = nibbles(np.asarray(codes_gpu).reshape(nblk, 16))
    cr = nibbles(np.asarray(codes_ref).reshape(nblk, 16))
    mis = (cg != cr) & keep[:, None]
    n_mis = int(np.count_nonzero(mis))
    exempt = 0
    if n_mis:
        bi, ei = np.nonzero(mis)
        e = sr[bi].astype(np.int64) - 127
        yr = y_ref.reshape(nblk, 32)[bi, ei].astype(np.float64)
        v = np.ldexp(yr, -e)
        w = REL * np.ldexp(ab.reshape(nblk, 32)[bi, ei], -e)
        near = np.abs(np.abs(v)[:, None] - BOUNDARIES[None, :]).min(axis=1) <= w
        near |= np.abs(v) <= w                         # sign of a zero
        exempt = int(np.count_nonzero(near))
    total_codes = nblk * 32
    res = {
        "blocks": nblk,
        "codes": total_codes,
        "scale_mismatch_unflagged": scale_bad,
        "scale_mismatch_flagged": scale_flagged_mis,
        "flagged_blocks": int(np.count_nonzero(flagged)),
        "code_mismatch": n_mis,
        "code_mismatch_exempt": exempt,
        "code_mismatch_nonexempt": n_mis - exempt,
    }
    res["ok"] = (scale_bad == 0 and res["code_mismatch_nonexempt"] == 0
                 and exempt <= allowed(total_codes)
                 and scale_flagged_mis <= allowed(nblk))
    return res


def check_exact(codes_gpu, scales_gpu, codes_ref, scales_ref):
    cg = np.asarray(codes_gpu)
    sg = np.asarray(scales_gpu)
    res = {
        "scale_mismatch": int(np.count_nonzero(sg != np.asarray(scales_ref))),
        "code_byte_mismatch": int(np.count_nonzero(cg != np.asarray(codes_ref))),
    }
    res["ok"] = res["scale_mismatch"] == 0 and res["code_byte_mismatch"] == 0
    return res
