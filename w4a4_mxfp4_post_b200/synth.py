"""Seeded synthetic inputs shaped like diffusion-transformer layer activations.

This module is the one piece that both the CUDA path and the CPU oracle are
fed from: it draws activations, Kronecker factors, SmoothQuant multipliers and
weights from seeded numpy generators.  It contains none of the quantizer's
arithmetic (no transform, no scale rule, no rounding to FP4).

Workloads (the shapes of the layer inputs of the models KroQuant evaluates,
"KroQuant ..." (arXiv 2607.21446), abstract: PixArt-Sigma, SANA, FLUX.1-schnell;
the trained models and datasets are not available, so seeded value models with
per-channel outliers stand in for real activations):

  tiny    64 x 128, N(0,1) x channel LogN(0,0.5), 2 outlier channels x40
  pixart  8192 x {1152, 4608}, N(0,1) x channel LogN(0,1) x token LogN(0,0.3),
          ceil(0.5% d) outlier channels x50
  sana    2048 x {2240, 5600}, Student-t(3) x channel LogN(0,1) x token
          LogN(0,0.3), ceil(0.5% d) outlier channels x100, shared factors
  flux    4608 x {3072, 12288}, the pixart base model; the last M//9 rows are
          "text" tokens (512 of 4608) and text and image rows each get their own
          ceil(1% d) outlier channels x80
  sweep   M in {256, 1024, 4096, 16384, 65536} x d in {1152, 3072, 12288}, the
          pixart value model

Random streams: channel-level draws come from SeedSequence([seed, 0]); rows
are drawn in chunks of ROW_CHUNK rows, chunk c from SeedSequence([seed, 1, c]),
so any row range can be regenerated on its own.  Factors use
SeedSequence([seed + 1000, 2]).
"""
from __future__ import annotations

import math

import numpy as np

ROW_CHUNK = 2048

WORKLOADS = {
    "tiny": {"M": 64, "ds": (128,), "model": "tiny", "factors": "per_block", "seed": 0},
    "pixart": {"M": 8192, "ds": (1152, 4608), "model": "pixart", "factors": "per_block", "seed": 1},
    "sana": {"M": 2048, "ds": (2240, 5600), "model": "sana", "factors": "shared", "seed": 2},
    "flux": {"M": 4608, "ds": (3072, 12288), "model": "flux", "factors": "per_block", "seed": 3},
    "sweep": {"Ms": (256, 1024, 4096, 16384, 65536), "ds": (1152, 3072, 12288),
              "model": "pixart", "factors": "per_block", "seed": 4},
}

MODELS = ("tiny", "pixart", "sana", "flux")

# The W4A4 linear layers fed by the quantizer: the PixArt-Sigma MLP at 8192
# tokens, (N, K) per layer: fc1 1152 -> 4608 and fc2 4608 -> 1152.
GEMM_LAYERS = {"pixart_mlp": {"M": 8192, "layers": ((4608, 1152), (1152, 4608)), "seed": 5}}


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-to-nearest-even) and return the raw bits."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """The float32 values of raw bf16 bits (exact: bf16 is the top half of binary32)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _channel_params(model: str, d: int, seed: int):
    g = _rng(seed, 0)
    if model == "tiny":
        ch = np.exp(0.5 * g.standard_normal(d))
        idx = g.choice(d, size=2, replace=False)
        ch[idx] *= 40.0
        return {"ch": ch}
    if model in ("pixart", "sana"):
        ch = np.exp(g.standard_normal(d))
        n_out = math.ceil(0.005 * d)
        idx = g.choice(d, size=n_out, replace=False)
        ch[idx] *= 50.0 if model == "pixart" else 100.0
        return {"ch": ch}
    if model == "flux":
        ch = np.exp(g.standard_normal(d))
        n_out = math.ceil(0.01 * d)
        img = g.choice(d, size=n_out, replace=False)
        txt = g.choice(d, size=n_out, replace=False)
        ch_img = ch.copy()
        ch_img[img] *= 80.0
        ch_txt = ch.copy()
        ch_txt[txt] *= 80.0
        return {"ch_img": ch_img, "ch_txt": ch_txt}
    raise ValueError(f"unknown value model {model!r}")


def _chunk_f32(model: str, M: int, d: int, seed: int, c: int, params) -> np.ndarray:
    r0 = c * ROW_CHUNK
    r1 = min(M, r0 + ROW_CHUNK)
    n = r1 - r0
    g = _rng(seed, 1, c)
    if model == "sana":
        z = g.standard_t(3.0, size=(n, d)).astype(np.float32)
    else:
        z = g.standard_normal((n, d), dtype=np.float32)
    if model == "tiny":
        z *= params["ch"].astype(np.float32)[None, :]
        return z
    tok = np.exp(0.3 * g.standard_normal(n)).astype(np.float32)
    if model == "flux":
        n_text = M // 9
        first_text = M - n_text
        img = slice(0, max(0, min(n, first_text - r0)))
        txt = slice(img.stop, n)
        z[img] *= params["ch_img"].astype(np.float32)[None, :]
        z[txt] *= params["ch_txt"].astype(np.float32)[None, :]
    else:
        z *= params["ch"].astype(np.float32)[None, :]
    z *= tok[:, None]
    return z


def activation(model: str, M: int, d: int, seed: int, rows: tuple[int, int] | None = None) -> np.ndarray:
    """bf16 activation bits [M, d] (uint16), or only rows [r0, r1) of it."""
    if d % 32 != 0 or d <= 0 or M < 0:
        raise ValueError("need M >= 0 and d a positive multiple of 32")
    r0, r1 = (0, M) if rows is None else rows
    if not (0 <= r0 <= r1 <= M):
        raise ValueError("row range out of bounds")
    params = _channel_params(model, d, seed)
    out = np.empty((r1 - r0, d), np.uint16)
    if r1 == r0:
        return out
    for c in range(r0 // ROW_CHUNK, (r1 - 1) // ROW_CHUNK + 1):
        cr0 = c * ROW_CHUNK
        block = bf16_bits_from_f32(_chunk_f32(model, M, d, seed, c, params))
        lo = max(r0, cr0)
        hi = min(r1, cr0 + block.shape[0])
        out[lo - r0:hi - r0] = block[lo - cr0:hi - cr0]
    return out


def factors(nb: int, seed: int, shared: bool = False) -> np.ndarray:
    """Kronecker factors [n, 5, 2, 2] float32 (n = 1 if shared else nb).

    Each 2x2 factor is I + 0.3 N(0,1), drawn again while |det| < 0.2.
    """
    g = _rng(seed + 1000, 2)
    n = 1 if shared else nb
    out = np.empty((n, 5, 2, 2), np.float32)
    for j in range(n):
        for k in range(5):
            while True:
                f = (np.eye(2) + 0.3 * g.standard_normal((2, 2))).astype(np.float32)
                if abs(float(f[0, 0]) * f[1, 1] - float(f[0, 1]) * f[1, 0]) >= 0.2:
                    break
            out[j, k] = f
    return out


def lu_params(nb: int, seed: int, shared: bool = False, noise: float = 0.1) -> np.ndarray:
    """LU scalars [n, 5, 3] float32 = (a, b, c) per factor (n = 1 if shared else nb).

    A learned transform starts at the Hadamard initialisation (a = b = 1/sqrt 2,
    c = 1) and moves from there: each scalar gets noise * N(0,1) added; |a|
    is kept >= 0.2.
    """
    g = _rng(seed + 2000, 4)
    n = 1 if shared else nb
    base = np.array([1 / np.sqrt(2.0), 1 / np.sqrt(2.0), 1.0])
    out = (base[None, None, :] + noise * g.standard_normal((n, 5, 3))).astype(np.float32)
    a = out[..., 0]
    out[..., 0] = np.where(np.abs(a) < 0.2, np.copysign(np.float32(0.2), a), a)
    return out


def adaln(nsamples: int, d: int, seed: int):
    """AdaLN modulation vectors (gamma, beta), each float32 [nsamples, d]:
    gamma ~ 0.2 N(0,1), beta ~ 0.1 N(0,1) (conditioning of a diffusion step)."""
    g = _rng(seed + 3000, 5)
    gamma = (0.2 * g.standard_normal((nsamples, d))).astype(np.float32)
    beta = (0.1 * g.standard_normal((nsamples, d))).astype(np.float32)
    return gamma, beta


def sq_multipliers(x_bf16: np.ndarray, alpha: float = 0.5, floor: float = 1e-5) -> np.ndarray:
    """SmoothQuant per-channel multipliers m_c = 1/s_c, s_c = max(max_r |X_rc|, floor)^alpha.

    This is the baseline's offline calibration (weight-free form), an input to
    the SmoothQuant quantizer, computed in double and rounded to fp32.
    """
    a = np.zeros(x_bf16.shape[1], np.float64)
    for r0 in range(0, x_bf16.shape[0], ROW_CHUNK):
        blk = np.abs(bf16_bits_to_f32(x_bf16[r0:r0 + ROW_CHUNK]))
        a = np.maximum(a, blk.max(axis=0).astype(np.float64))
    s = np.maximum(a, floor) ** alpha
    return (1.0 / s).astype(np.float32)


def weights(N: int, d: int, seed: int) -> np.ndarray:
    """fp32 weights [N, d], N(0,1), for the fold check."""
    return _rng(seed, 3).standard_normal((N, d)).astype(np.float32)


def workload_layers(name: str):
    """(M, d, model, shared, seed) for every layer input of a named workload."""
    w = WORKLOADS[name]
    shared = w["factors"] == "shared"
    Ms = w.get("Ms", (w.get("M"),))
    return [(M, d, w["model"], shared, w["seed"]) for M in Ms for d in w["ds"]]


def mx_operand(rows: int, K: int, seed: int, scale_lo: int = 112, scale_hi: int = 142):
    """A random MXFP4 operand: codes [rows, K/2] (every byte value equally
    likely, so every E2M1 code and sign) and E8M0 scale bytes [rows, K/32]
    uniform in [scale_lo, scale_hi)."""
    g = _rng(seed, 7, rows, K)
    codes = g.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = g.integers(scale_lo, scale_hi, (rows, K // 32), dtype=np.uint8)
    return codes, scales
