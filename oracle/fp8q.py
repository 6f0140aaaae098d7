"""Float64 CPU oracle of the FP8 (e4m3) variant of the block-sparse attention stage.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA path and must never be used
as a fallback for it.

The pages mention FP8 only for the deployment of the video model ([LF-yly] section 五:
weights quantised per channel and activations per token, "nearly lossless"; the
gist.science explainer, section 4: FP8 linear layers).  Applying FP8 to the attention
operands is an extension; its reading, stated here once:

  * format: OCP e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest
    finite value 448; subnormals m * 2^-9; no infinities), round to nearest, ties to the
    even code;
  * scales are powers of two, so that x / scale and x8 * scale are exact: the scale of a
    group of values is 2^e with e the smallest integer such that max|x| <= 448 * 2^e
    (1 for an all-zero group);
  * the queries are quantised per (token, head), as the page quantises activations per
    token; the keys per head (one scale over every key the call can attend to), so that a
    key tile of the attention needs no per-column factor;
  * the values stay bf16;
  * the attention is then exactly the block-sparse attention of the dequantised queries
    and keys (x8 * scale) with the bf16 values: hsa64.attention on those tensors.
"""
from __future__ import annotations

import numpy as np

__all__ = ["E4M3_MAX", "e4m3_positive_values", "round_e4m3", "pow2_scale_exponent",
           "quantize_rows", "quantize_per_head", "dequantize"]

E4M3_MAX = 448.0


def e4m3_positive_values():
    """(values, codes) of the non-negative finite e4m3 numbers, ascending: code 0..7 are
    the subnormals m * 2^-9 (m = 0..7), code 8*e + m (e = 1..15, m = 0..7, except the NaN
    code 0x7f) is (1 + m/8) * 2^(e - 7)."""
    vals, codes = [], []
    for m in range(8):
        vals.append(m * 2.0 ** -9)
        codes.append(m)
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
            codes.append(8 * e + m)
    return np.array(vals), np.array(codes, dtype=np.int64)


_VALS, _CODES = e4m3_positive_values()


def round_e4m3(v) -> np.ndarray:
    """Round |v| <= 448 to the nearest e4m3 value, ties to the even code; returns float64
    values on the e4m3 grid (the sign kept)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    if np.any(a > E4M3_MAX):
        raise ValueError("value above the e4m3 range")
    hi = np.searchsorted(_VALS, a, side="left")           # first grid value >= a
    hi = np.minimum(hi, len(_VALS) - 1)
    lo = np.maximum(hi - 1, 0)
    exact = _VALS[hi] == a
    d_lo, d_hi = a - _VALS[lo], _VALS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_CODES[hi] % 2 == 0))
    idx = np.where(exact, hi, np.where(pick_hi, hi, lo))
    return np.copysign(_VALS[idx], v)


def pow2_scale_exponent(amax: float) -> int:
    """The smallest integer e with amax <= 448 * 2^e (0 for amax == 0)."""
    amax = float(amax)
    if amax == 0.0:
        return 0
    e = int(np.ceil(np.log2(amax / E4M3_MAX)))
    while amax > E4M3_MAX * 2.0 ** e:
        e += 1
    while amax <= E4M3_MAX * 2.0 ** (e - 1):
        e -= 1
    return e


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        import torch
        return x.detach().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def quantize_rows(x):
    """x [..., d] -> (x8 [..., d] e4m3 values, scale [...]): one power-of-two scale per
    row of the last axis (per (token, head) for a [tokens, H, d] tensor)."""
    x = _f64(x)
    amax = np.abs(x).max(axis=-1)
    e = np.vectorize(pow2_scale_exponent, otypes=[np.int64])(amax)
    scale = np.ldexp(1.0, e)
    return round_e4m3(x / scale[..., None]), scale


def quantize_per_head(x, head_axis: int = -2):
    """x [..., H, d] -> (x8, scale [H]): one power-of-two scale per head over every other
    axis."""
    x = _f64(x)
    xm = np.moveaxis(x, head_axis, 0)
    H = xm.shape[0]
    scale = np.array([np.ldexp(1.0, pow2_scale_exponent(np.abs(xm[h]).max())) for h in range(H)])
    shape = [1] * x.ndim
    shape[head_axis] = H
    return round_e4m3(x / scale.reshape(shape)), scale


def dequantize(x8, scale, axis_shape=None) -> np.ndarray:
    """x8 * scale with the scale broadcast over the quantised group (exact)."""
    x8 = np.asarray(x8, dtype=np.float64)
    scale = np.asarray(scale, dtype=np.float64)
    if axis_shape is not None:
        scale = scale.reshape(axis_shape)
    return x8 * scale
