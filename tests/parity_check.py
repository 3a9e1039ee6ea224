"""Agreement criteria between the CUDA path and the CPU oracle.

KroQuant quantizer (transform + MXFP4), with y_ref the oracle's fp32 transform
and ab = |K||x| (the scale of a dot product's rounding error):

  transform  |y_gpu - y_ref| <= 1e-5 * ab                    (relative error
             taken against |K||x|, the standard dot-product error scale; a
             per-element relative test is ill-posed where y ~ 0)
  scales     bit-exact, except in "flagged" blocks, whose oracle amax lies
             within the transform tolerance of a power of two (a legitimate
             fp32 evaluation may then take the neighbouring exponent): any
             unflagged mismatch fails the case; flagged mismatches are counted
             (their blocks' codes are not compared) and bounded as a rate over
             ALL compared blocks, like the exempt codes below.
  codes      bit-exact, except where the oracle's scaled value v = y_ref 2^-e
             lies within w = 1e-5 * ab * 2^-e of a rounding boundary of E2M1
             (+-0.25, +-0.75, ..., +-5, or 0 for the sign of a zero); such
             "exempt" mismatches are counted.  Any other mismatch fails the
             case.  The exempt count is bounded as a rate over ALL compared
             codes: the cases of a test session add their counts to POOL, and
             pooled_verdict() requires sum(exempt) <= 1e-6 * sum(codes) and
             sum(flagged scale mismatches) <= 1e-6 * sum(blocks).

  Of the exempt mismatches, those whose v is NOT within 1e-5 * b of the
  nearest boundary b (the boundary-relative window) are reported separately
  as `code_mismatch_exempt_outside_rel`: the window above is wider where the
  transform cancels (|y| << |K||x|), and a sign-of-zero flip (boundary 0) is
  always outside a boundary-relative window.

SmoothQuant and plain MXFP4: codes and scales bit-exact, no exemptions (the
fp32 product x * m is correctly rounded on both sides).
"""
from __future__ import annotations

import numpy as np

BOUNDARIES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
REL = 1e-5
EXEMPT_FRACTION = 1e-6

# Counts of every KroQuant-type case checked in this process (pool=True).
POOL = {"cases": 0, "codes": 0, "blocks": 0, "code_mismatch_exempt": 0,
        "code_mismatch_exempt_outside_rel": 0, "flagged_blocks": 0, "scale_mismatch_flagged": 0}


def nibbles(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def scale_band_flags(y_ref: np.ndarray, ab: np.ndarray) -> np.ndarray:
    """[nblocks] True where the block amax lies within the transform tolerance of a power of two."""
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


def check_kq(codes_gpu, scales_gpu, codes_ref, scales_ref, y_ref, ab, pool: bool = True):
    """Counts per the criteria above; `ok` is the per-case verdict.

    pool=False keeps the counts out of POOL (for checks of planted mismatches).
    """
    sg = np.asarray(scales_gpu).reshape(-1)
    sr = np.asarray(scales_ref).reshape(-1)
    nblk = sr.size
    flagged = scale_band_flags(y_ref, ab)
    smis = sg != sr
    cg = nibbles(np.asarray(codes_gpu).reshape(nblk, 16))
    cr = nibbles(np.asarray(codes_ref).reshape(nblk, 16))
    mis = (cg != cr) & ~smis[:, None]              # codes of blocks with equal scales
    n_mis = int(np.count_nonzero(mis))
    exempt = 0
    outside_rel = 0
    if n_mis:
        bi, ei = np.nonzero(mis)
        e = sr[bi].astype(np.int64) - 127
        yr = y_ref.reshape(nblk, 32)[bi, ei].astype(np.float64)
        v = np.abs(np.ldexp(yr, -e))
        w = REL * np.ldexp(ab.reshape(nblk, 32)[bi, ei], -e)
        dist = np.abs(v[:, None] - BOUNDARIES[None, :])
        near = (dist.min(axis=1) <= w) | (v <= w)      # a boundary, or the sign of a zero
        exempt = int(np.count_nonzero(near))
        near_rel = (dist <= REL * BOUNDARIES[None, :]).any(axis=1)
        outside_rel = int(np.count_nonzero(near & ~near_rel))
    total_codes = nblk * 32
    res = {
        "blocks": nblk,
        "codes": total_codes,
        "scale_mismatch": int(np.count_nonzero(smis)),
        "scale_mismatch_unflagged": int(np.count_nonzero(smis & ~flagged)),
        "scale_mismatch_flagged": int(np.count_nonzero(smis & flagged)),
        "flagged_blocks": int(np.count_nonzero(flagged)),
        "code_mismatch": n_mis,
        "code_mismatch_exempt": exempt,
        "code_mismatch_exempt_outside_rel": outside_rel,
        "code_mismatch_nonexempt": n_mis - exempt,
    }
    res["ok"] = res["scale_mismatch_unflagged"] == 0 and res["code_mismatch_nonexempt"] == 0
    if pool:
        POOL["cases"] += 1
        POOL["codes"] += total_codes
        POOL["blocks"] += nblk
        POOL["code_mismatch_exempt"] += exempt
        POOL["code_mismatch_exempt_outside_rel"] += outside_rel
        POOL["flagged_blocks"] += res["flagged_blocks"]
        POOL["scale_mismatch_flagged"] += res["scale_mismatch_flagged"]
    return res


def pooled_verdict(pool: dict | None = None) -> dict:
    """The rate criteria over every case pooled so far: exempt codes <= 1e-6
    of all compared codes, flagged scale mismatches <= 1e-6 of all blocks."""
    p = dict(POOL if pool is None else pool)
    p.setdefault("scale_mismatch_flagged", 0)
    p["exempt_rate"] = p["code_mismatch_exempt"] / p["codes"] if p["codes"] else 0.0
    p["exempt_outside_rel_rate"] = p["code_mismatch_exempt_outside_rel"] / p["codes"] if p["codes"] else 0.0
    p["scale_flagged_rate"] = p["scale_mismatch_flagged"] / p["blocks"] if p["blocks"] else 0.0
    p["ok"] = (p["code_mismatch_exempt"] <= EXEMPT_FRACTION * p["codes"]
               and p["scale_mismatch_flagged"] <= EXEMPT_FRACTION * p["blocks"])
    return p


def check_exact(codes_gpu, scales_gpu, codes_ref, scales_ref):
    cg = np.asarray(codes_gpu)
    sg = np.asarray(scales_gpu)
    res = {
        "scale_mismatch": int(np.count_nonzero(sg != np.asarray(scales_ref))),
        "code_byte_mismatch": int(np.count_nonzero(cg != np.asarray(codes_ref))),
    }
    res["ok"] = res["scale_mismatch"] == 0 and res["code_byte_mismatch"] == 0
    return res


# -- the W4A4 product ---------------------------------------------------------------
# Each product of two MXFP4 values is exact (two significant bits times a power
# of two), so the product differs from the oracle's double sum only by the fp32
# accumulation: per element at most K * 2^-23 * sum_k |a_k b_k| (any order,
# truncating adds included), plus bf16's rounding of the output (2^-8 of the
# value).  That worst case grows with K; accumulation errors of random sign
# grow with sqrt(K), so the fp32 results must also meet a statistical bound:
# the root mean square over all elements of err / sum_k |a_k b_k| at most
# GEMM_RMS_FACTOR * sqrt(K) * 2^-24.  A systematic mistake that the per-element
# bound could miss (a dropped or repeated K-block, whose contribution is a
# near-cancelling partial sum) moves this statistic by orders of magnitude.
GEMM_RMS_FACTOR = 8.0


def gemm_bound(K, D, absd, bf16_out):
    acc = K * 2.0 ** -23 * absd
    return acc + (2.0 ** -8 * (np.abs(D) + acc) if bf16_out else 0.0)


def check_gemm(Dg, D, absd, K, bf16_out):
    """Per-element worst-case bound; for fp32 output also the rms statistic.

    Returns {"bad": elements over the bound, "worst": max err / bound,
    "rms_rel": rms of err / absd (fp32 only), "rms_bound": its bound, "ok"}."""
    err = np.abs(np.asarray(Dg, np.float64) - D)
    bound = gemm_bound(K, D, absd, bf16_out)
    bad = int(np.count_nonzero(err > bound))
    res = {"bad": bad, "worst": float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0}
    ok = bad == 0
    if not bf16_out:
        nz = absd > 0
        rel = err[nz] / absd[nz]
        res["rms_rel"] = float(np.sqrt(np.mean(rel * rel))) if rel.size else 0.0
        res["rms_bound"] = GEMM_RMS_FACTOR * np.sqrt(K) * 2.0 ** -24
        ok = ok and res["rms_rel"] <= res["rms_bound"]
    res["ok"] = ok
    return res
