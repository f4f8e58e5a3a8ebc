"""FP8 scores with incoherent processing: the plain fp64 definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

"FlashAttention-3 …" (FlashAttention-3의 기술적 혁신, item 3: low precision
with reduced quantisation error) describes the method: before the scores
are formed, the query and key feature vectors are multiplied by a random
orthogonal matrix such as a Hadamard matrix; the rotation spreads
outlier coordinates over all coordinates, so that quantising to FP8 loses
less; and, the rotation being orthogonal, it cancels in Q K^T.  The pages
fix neither the FP8 format's details nor the scale granularity nor whether
V and P are quantised too.  Readings:

* the rotation is R = diag(sigma) H_D / sqrt(D): H_D the Sylvester Hadamard
  matrix of order D (a power of two), sigma a vector of D random signs
  (an input, drawn by the caller);
* FP8 is OCP e4m3 ("e4m3fn": 4 exponent bits with bias 7, 3 mantissa bits,
  no infinities, largest finite value 448, subnormals down to 2^-9),
  rounded to nearest with ties to even, saturating at +-448;
* each (b, head) of the rotated Q and of the rotated K has one scale, its
  absolute maximum / 448; the stored values are e4m3(x / scale);
* only Q K^T is formed from FP8 values (the step the pages rotate); the
  softmax, its mods and P V follow the exact definition of ``attention``.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_forward

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6     # 2^(1 - bias)
E4M3_MANTISSA_BITS = 3


def hadamard(D: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order D (entries +-1): H_1 = [1],
    H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    if D < 1 or D & (D - 1):
        raise ValueError("D must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < D:
        H = np.block([[H, H], [H, -H]])
    return H


def rotation(D: int, signs) -> np.ndarray:
    """The orthonormal rotation diag(signs) H_D / sqrt(D)."""
    signs = np.asarray(signs, dtype=np.float64)
    if signs.shape != (D,) or not np.all(np.abs(signs) == 1.0):
        raise ValueError("signs must be D values of +-1")
    return signs[:, None] * hadamard(D) / np.sqrt(D)


def quantize_e4m3(x) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to even, saturating at +-448.
    Each binade [2^e, 2^(e+1)) holds 8 values spaced 2^(e-3); below the
    smallest normal (2^-6) the spacing stays 2^-9 (subnormals)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, E4M3_MIN_NORMAL_EXP)
    quantum = np.exp2(e - E4M3_MANTISSA_BITS)
    q = np.round(a / quantum) * quantum          # numpy rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, x)


def quantize_per_head(x):
    """Per (b, head) absmax scaling to e4m3: returns (values on the e4m3 grid,
    scales [B][H]); x ~ values * scale.  An all-zero head gets scale 1."""
    amax = np.abs(x).max(axis=(2, 3))
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return quantize_e4m3(x / scale[:, :, None, None]), scale


def fwht(x):
    """The fast Walsh-Hadamard transform along the last axis, in the dtype of
    x: stages h = 1, 2, 4, ..., D/2, each replacing the pair (y[i], y[i + h])
    of every block of 2h by (y[i] + y[i + h], y[i] - y[i + h]).  Equals
    x @ hadamard(D) (the Sylvester matrix is symmetric)."""
    y = np.array(x, copy=True)
    D = y.shape[-1]
    if D < 1 or D & (D - 1):
        raise ValueError("D must be a power of two")
    h = 1
    while h < D:
        y = y.reshape(*y.shape[:-1], D // (2 * h), 2, h)
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :], y[..., 1, :] = a + b, a - b
        y = y.reshape(*y.shape[:-3], D)
        h *= 2
    return y


def prep_fp32(x, signs):
    """The rotation and per-head quantisation in fp32, one operation at a
    time, as a kernel computes them: y = fwht(x * signs) * (1 / sqrt(D))
    (one fp32 product by the fp32 constant), amax per (b, head), scale =
    amax / 448, codes = e4m3(y / scale) with IEEE fp32 division.  Every
    step is an exactly rounded fp32 operation, so a kernel that takes the
    same steps gets the same codes.  Returns (codes as float64, scales)."""
    x = np.asarray(x, dtype=np.float32)
    D = x.shape[-1]
    inv_sqrt_d = np.float32(1.0 / np.sqrt(D))
    y = fwht(x * np.asarray(signs, dtype=np.float32)) * inv_sqrt_d
    amax = np.abs(y).max(axis=(2, 3))
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    ratio = (y / scale[:, :, None, None]).astype(np.float32)
    return quantize_e4m3(ratio.astype(np.float64)), scale.astype(np.float64)


def attention_forward_fp8(q, k, v, scale, signs=None, mod=0, params=None, heads=None, rows=None):
    """O and LSE with the scores formed from FP8 Q and K.

    signs: D random signs of the incoherent-processing rotation, or None to
    quantise Q and K as they are (the un-rotated FP8 baseline).
    Returns (O, LSE) like ``attention_forward``.
    """
    D = q.shape[-1]
    if signs is not None:
        R = rotation(D, signs)
        q, k = q @ R, k @ R
    q8, sq = quantize_per_head(q)
    k8, sk = quantize_per_head(k)
    # dequantised FP8 operands: the scores are exactly scale * (q8 sq) . (k8 sk)
    return attention_forward(q8 * sq[:, :, None, None], k8 * sk[:, :, None, None], v, scale, mod, params,
                             heads=heads, rows=rows)
