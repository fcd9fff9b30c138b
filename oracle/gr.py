"""Gated Residual (GR) read and write with an FP8 residual state: slow, plain
numpy reference (test infrastructure only; only the tests, the smoke check
and the benchmark's CPU-baseline leg may use it).

What it computes ("Qwen3.8-Flash-Next: architecture, efficiency and technical
lineage", section 05 "Residual design", part 4 "GR" and its "Group RMSNorm",
"Low-rank router" and "No Hres" boxes; the inference paragraph of the same
section for the FP8 state and the fused read/write):

  R^_i = RMSNorm(R_i; gamma_i)                       each of the n_r branches
  G    = unvec(sigmoid(W_u SiLU((1/n_r) W_d vec(R^))))    n_r x d gates
  x    = (1/n_r) sum_i G_i o R^_i                     the block input (read)
  s    = 2 sigmoid((1/n_r) W_w vec(R^))               n_r write scalars in (0, 2)
  R'_i = R_i + s_i y                                  the write of block output y

Readings where the pages are silent (listed in the design notes):
  * RMSNorm(r; gamma) = r / sqrt(mean(r^2) + eps) * gamma, eps = 1e-6;
  * the FP8 state is OCP E4M3 (finite-saturating, round to nearest even) with
    one fp32 scale per (token, branch) row: value = decode(code) * scale, and
    a written row takes scale = max|R'| / 448 (1 when the row is all zero);
  * s is passed from the read to the write (it is a function of the state
    before the block, which the read has at hand).

Read: fp64 arithmetic from the exact fp32 dequantised state.  Write: the
new state R' = R + s y is an fp32 row (the state's own precision), formed with
one rounding per operation: r = deq + s * y (product rounded, then the sum).
The row's scale is amax / 448 rounded to fp32.  Each code is the E4M3 value
nearest to the exact quotient r / scale (ties to the even code), i.e. one
rounding from the definition of the format; the quotient is taken in fp64,
which is exact enough: for fp32 r and scale, r / scale is either an E4M3
rounding boundary itself or at least 2^-29 (relative) away from every
boundary, so the fp64 quotient (relative error 2^-53) rounds the same way.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Value of each E4M3 code (uint8) as float64: sign, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6);
    S.1111.111 is NaN; there are no infinities."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # codes 0x00..0x7E, increasing


def e4m3_encode(x):
    """Round float values to E4M3 codes: nearest representable value, ties to
    the even code (even mantissa), magnitudes above 448 saturate to 448, the
    sign of zero is kept, NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # index of the largest representable value <= a (a >= 0)
    lo = np.clip(np.searchsorted(_POS, a, side="right") - 1, 0, len(_POS) - 1)
    hi = np.clip(lo + 1, 0, len(_POS) - 1)
    dlo = a - _POS[lo]
    dhi = _POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def dequant(codes, scales):
    """fp32 state: decode(code) * scale, one fp32 rounding, as the kernels do.
    codes [..., n_r, d] uint8; scales [..., n_r] fp32."""
    v = e4m3_decode(codes).astype(np.float32)
    return (v * np.asarray(scales, np.float32)[..., None]).astype(np.float32)


def quantize_rows(r):
    """fp32 rows [..., d] -> (codes uint8, scales fp32): the row's own scale
    amax / 448 rounded to fp32 (1 for an all-zero row), and code = the E4M3
    value nearest to the exact quotient r / scale (see the module notes on
    why an fp64 quotient gives the same rounding)."""
    r = np.asarray(r, dtype=np.float32)
    amax = np.abs(r).max(axis=-1).astype(np.float32)
    scale = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32),
                     np.float32(1.0)).astype(np.float32)
    q = r.astype(np.float64) / scale.astype(np.float64)[..., None]
    return e4m3_encode(q), scale


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def gr_read(codes, scales, gamma, W_d, W_u, W_w, eps=1e-6, parts=False):
    """GR read.  codes [T, n_r, d] uint8, scales [T, n_r] fp32; gamma [n_r, d];
    W_d [r, n_r d], W_u [n_r d, r], W_w [n_r, n_r d] (any float dtype; used
    exactly).  Returns (x [T, d], s [T, n_r]) in fp64, and with parts=True
    also a dict of R^, h, G."""
    R = dequant(codes, scales).astype(np.float64)
    T, n_r, d = R.shape
    ms = (R * R).mean(axis=-1, keepdims=True)
    Rh = R / np.sqrt(ms + eps) * np.asarray(gamma, np.float64)[None]
    z = Rh.reshape(T, n_r * d)
    Wd = np.asarray(W_d, np.float64)
    Wu = np.asarray(W_u, np.float64)
    Ww = np.asarray(W_w, np.float64)
    a = (z @ Wd.T) / n_r
    h = a * _sigmoid(a)                       # SiLU
    G = _sigmoid(h @ Wu.T).reshape(T, n_r, d)
    x = (G * Rh).sum(axis=1) / n_r
    s = 2.0 * _sigmoid((z @ Ww.T) / n_r)
    if parts:
        return x, s, dict(rhat=Rh, h=h, G=G)
    return x, s


def gr_write(codes, scales, y, s):
    """GR write: R'_i = R_i + s_i y, requantised per row.  codes [T, n_r, d]
    uint8, scales [T, n_r] fp32, y [T, d] (bf16 values, any float dtype), s
    [T, n_r] fp32.  Returns (codes', scales') with every step in fp32."""
    R = dequant(codes, scales)
    y32 = np.asarray(y, np.float32)
    s32 = np.asarray(s, np.float32)
    prod = (s32[..., None] * y32[:, None, :]).astype(np.float32)
    r = (R + prod).astype(np.float32)
    return quantize_rows(r)
