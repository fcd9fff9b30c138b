"""Pins for the Gated Residual oracle (oracle/gr.py): "Qwen3.8-Flash-Next:
architecture, efficiency and technical lineage", section 05 "Residual
design", part 4 "GR" (read and write formulas, "Group RMSNorm",
"Low-rank router") and the FP8 residual state of the same section.

* E4M3 codec against the format's definition: known codes (1.0, 448, the
  smallest normal and subnormal, -0), every finite code round-trips,
  midpoints round to the even code, saturation at 448;
* read with a zero router (W_d = 0 or W_u = 0): every gate is 1/2, so
  x = (1/2 n_r) sum_i R^_i; with W_w = 0 every write scalar is 1;
* one branch with a saturated router (W_u huge): x = R^, the plain pre-norm
  read that GR replaces;
* RMSNorm: each R^_i has mean square 1 for gamma = 1 (eps = 0), and the read
  is invariant to rescaling a branch's state;
* write: y = 0 leaves the dequantised state unchanged up to requantisation;
  a zero state takes the quantised s y.
"""
import numpy as np
import pytest

from oracle import gr


def test_e4m3_known_codes():
    v = gr.e4m3_decode(np.array([0x38, 0x7E, 0x08, 0x01, 0x80, 0x00, 0x07, 0xBE, 0x7F],
                                np.uint8))
    assert v[0] == 1.0 and v[1] == 448.0 and v[2] == 2.0 ** -6 and v[3] == 2.0 ** -9
    assert v[4] == 0.0 and np.signbit(v[4]) and v[5] == 0.0 and not np.signbit(v[5])
    assert v[6] == 7 / 8 * 2.0 ** -6 and v[7] == -(1.75 * 2.0 ** 0) and np.isnan(v[8])


def test_e4m3_round_trip_ties_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    np.testing.assert_array_equal(gr.e4m3_encode(gr.e4m3_decode(codes)), codes)
    # midpoints between neighbours go to the even code
    pos = gr.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    got = gr.e4m3_encode(mids)
    want = np.where(np.arange(len(mids)) % 2 == 0, np.arange(len(mids)),
                    np.arange(len(mids)) + 1)
    np.testing.assert_array_equal(got, want)
    assert gr.e4m3_encode(np.array([449.0, 1e6, -500.0])).tolist() == [0x7E, 0x7E, 0xFE]
    assert gr.e4m3_encode(np.array([2.0 ** -11]))[0] == 0  # below half the smallest subnormal


def _state(T, n_r, d, seed):
    r = np.random.default_rng(seed)
    R = (r.standard_normal((T, n_r, d)) * r.uniform(0.5, 4.0, (T, n_r, 1))).astype(np.float32)
    return gr.quantize_rows(R)


def _weights(n_r, d, rank, seed, scale=0.05):
    r = np.random.default_rng(seed)
    return (r.standard_normal((n_r, d)) * 0.1 + 1.0, r.standard_normal((rank, n_r * d)) * scale,
            r.standard_normal((n_r * d, rank)) * scale, r.standard_normal((n_r, n_r * d)) * scale)


def test_zero_router_gives_half_gates_and_unit_writes():
    codes, scales = _state(6, 4, 32, 1)
    gamma, Wd, Wu, Ww = _weights(4, 32, 4, 2)
    for wd, wu in ((0 * Wd, Wu), (Wd, 0 * Wu)):
        x, s, p = gr.gr_read(codes, scales, gamma, wd, wu, 0 * Ww, parts=True)
        np.testing.assert_allclose(p["G"], 0.5, rtol=0, atol=0)
        np.testing.assert_allclose(x, p["rhat"].sum(axis=1) / 8, rtol=1e-14, atol=1e-14)
        np.testing.assert_array_equal(s, 1.0)


def test_single_branch_saturated_router_is_the_prenorm_read():
    """n_r = 1 with a positive state and a positive router: every gate is
    sigmoid(>= 40) = 1 in fp64, so the read is R^ itself."""
    r = np.random.default_rng(3)
    R = np.abs(r.standard_normal((5, 1, 16))).astype(np.float32) + 0.1
    codes, scales = gr.quantize_rows(R)
    gamma = np.ones((1, 16))
    Wd = np.full((2, 16), 0.5)
    Wu = np.full((16, 2), 1e3)
    x, _, p = gr.gr_read(codes, scales, gamma, Wd, Wu, np.zeros((1, 16)), parts=True)
    assert (p["h"] > 0.04).all()
    np.testing.assert_array_equal(p["G"], 1.0)
    np.testing.assert_allclose(x, p["rhat"][:, 0], rtol=1e-15, atol=0)


def test_rmsnorm_and_scale_invariance():
    codes, scales = _state(4, 4, 64, 5)
    _, Wd, Wu, Ww = _weights(4, 64, 8, 6)
    one = np.ones((4, 64))
    x, s, p = gr.gr_read(codes, scales, one, Wd, Wu, Ww, eps=0.0, parts=True)
    np.testing.assert_allclose((p["rhat"] ** 2).mean(axis=-1), 1.0, rtol=1e-12)
    # a branch's state scaled by 2 (an exact change of its scale) reads the same
    scales2 = scales.copy()
    scales2[:, 1] *= 2
    x2, s2 = gr.gr_read(codes, scales2, one, Wd, Wu, Ww, eps=0.0)
    np.testing.assert_allclose(x2, x, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s, rtol=1e-12, atol=1e-13)


def test_write_closed_forms():
    codes, scales = _state(3, 4, 32, 7)
    y = np.random.default_rng(8).standard_normal((3, 32)).astype(np.float32)
    s = np.random.default_rng(9).uniform(0.1, 1.9, (3, 4)).astype(np.float32)
    # y = 0: the dequantised state, requantised per row
    c0, sc0 = gr.gr_write(codes, scales, np.zeros_like(y), s)
    want_c, want_s = gr.quantize_rows(gr.dequant(codes, scales))
    np.testing.assert_array_equal(c0, want_c)
    np.testing.assert_array_equal(sc0, want_s)
    # a zero state: the quantised s y
    z = np.zeros_like(codes)
    c1, sc1 = gr.gr_write(z, np.ones_like(scales), y, s)
    want_c, want_s = gr.quantize_rows((s[..., None] * y[:, None, :]).astype(np.float32))
    np.testing.assert_array_equal(c1, want_c)
    np.testing.assert_array_equal(sc1, want_s)
    # dequantised result is within half an E4M3 step (relative 2^-4) of the exact sum
    c2, sc2 = gr.gr_write(codes, scales, y, s)
    exact = gr.dequant(codes, scales).astype(np.float64) + s[..., None] * y[:, None, :]
    got = gr.dequant(c2, sc2)
    np.testing.assert_array_less(np.abs(got - exact), np.abs(exact) * 2.0 ** -4 + sc2[..., None] * 2.0 ** -9)


def test_identical_branches_read_as_one():
    """n_r copies of one branch, with the router and write weights repeated
    block by block, read exactly as that single branch: pins every 1/n_r
    factor and the vec/unvec ordering."""
    codes1, scales1 = _state(7, 1, 24, 11)
    gamma1, Wd1, Wu1, Ww1 = _weights(1, 24, 3, 12, scale=0.3)
    x1, s1, p1 = gr.gr_read(codes1, scales1, gamma1, Wd1, Wu1, Ww1, parts=True)
    n = 4
    codes = np.repeat(codes1, n, axis=1)
    scales = np.repeat(scales1, n, axis=1)
    gamma = np.repeat(gamma1, n, axis=0)
    Wd = np.tile(Wd1, (1, n))        # [r, n d]: the same block for every branch
    Wu = np.tile(Wu1, (n, 1))        # [n d, r]
    Ww = np.tile(Ww1, (n, n))        # [n, n d]
    x, s, p = gr.gr_read(codes, scales, gamma, Wd, Wu, Ww, parts=True)
    np.testing.assert_allclose(x, x1, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s, np.repeat(s1, n, axis=1), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(p["G"], np.repeat(p1["G"], n, axis=1), rtol=1e-13, atol=1e-14)


def _nearest_code_exact(r, s):
    """The E4M3 code nearest to the exact rational r / s (ties to the even
    code, saturating at 448), by brute force over the code table with
    fractions.Fraction: independent of the oracle's fp64 quotient."""
    from fractions import Fraction
    q = Fraction(float(r)) / Fraction(float(s))
    a = abs(q)
    pos = gr.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    if a >= 448:
        c = 0x7E
    else:
        best = None
        for code in range(0x7F):
            dist = abs(a - Fraction(float(pos[code])))
            if best is None or dist < best[0] or (dist == best[0] and code % 2 == 0):
                best = (dist, code)
        c = best[1]
    return c | (0x80 if q < 0 or (q == 0 and np.signbit(r)) else 0)


# Rows (amax, r) found by search where the fp32 reciprocal form
# E4M3(r * fl(1 / scale)) and the exact E4M3(r / scale) fall on opposite
# sides of a rounding boundary, in both directions.  Bit patterns of the fp32
# values, with the reciprocal form's code and the exact code.
_TIE_ROWS = [
    (1085189614, 1024425110, 68, 67),
    (1067759192, 976641066, 40, 39),
    (1066323723, 964625409, 28, 29),
]


def test_quantize_rounds_the_exact_quotient():
    """The written code is the E4M3 rounding of the exact quotient r / scale
    (the format's definition), not of an fp32 reciprocal product: pinned on
    rows where the two differ, and on a random sample against brute force."""
    for amax_bits, r_bits, recip_code, exact_code in _TIE_ROWS:
        amax = np.array([amax_bits], np.uint32).view(np.float32)[0]
        r = np.array([r_bits], np.uint32).view(np.float32)[0]
        row = np.array([[amax, r, -r]], np.float32)
        codes, scales = gr.quantize_rows(row)
        s = scales[0]
        assert s == np.float32(amax / np.float32(448.0))
        inv = np.float32(np.float32(1.0) / s)
        # the reciprocal form really does round the other way here
        assert int(gr.e4m3_encode(np.array([np.float32(r * inv)], np.float64))[0]) == recip_code
        assert _nearest_code_exact(r, s) == exact_code != recip_code
        assert int(codes[0, 1]) == exact_code
        assert int(codes[0, 2]) == exact_code | 0x80
        assert int(codes[0, 0]) == 0x7E
    rng = np.random.default_rng(21)
    R = (rng.standard_normal((6, 40)) * rng.uniform(0.01, 50.0, (6, 1))).astype(np.float32)
    R[0, :5] = 0.0
    R[1, 3] = -0.0
    codes, scales = gr.quantize_rows(R)
    for i in range(R.shape[0]):
        for j in range(R.shape[1]):
            assert int(codes[i, j]) == _nearest_code_exact(R[i, j], scales[i]), (i, j)
