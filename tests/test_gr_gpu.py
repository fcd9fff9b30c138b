"""Gated Residual read and write on the GPU against the oracle (oracle/gr.py).

Read: x and s within the bf16 bar (the router and the write scalars come
from bf16 GEMMs with fp32 accumulation; R^, the router output and the logits
are held in bf16).
Write: the E4M3 codes (the rounding of the exact quotient r / scale) and the
scales are integers / floats decided by fp32
arithmetic in a fixed order, so they must match the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

from gated_deltanet_scan_chunked_b200 import gdn, gdn_check_device_error, inputs
from oracle import gr as ogr
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _np(x):
    return x.detach().to("cpu").float().numpy() if x.dtype != torch.uint8 else x.cpu().numpy()


def _cuda(g):
    return {k: v.cuda() for k, v in g.items()}


@pytest.mark.parametrize("T,n_r,d,rank", [(300, 4, 256, 32), (128, 4, 2560, 320), (17, 1, 64, 8),
                                          (64, 3, 128, 16), (40, 8, 96, 24)])
def test_gr_read(T, n_r, d, rank):
    g = inputs.make_gr(T, n_r, d, rank, seed=T + d)
    c = _cuda(g)
    x, s = gdn.gdn_gr_read(c["codes"], c["scales"], c["gamma"], c["W_d"], c["W_u"], c["W_w"])
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    xr, sr = ogr.gr_read(_np(g["codes"]), _np(g["scales"]), _np(g["gamma"]), _np(g["W_d"]),
                         _np(g["W_u"]), _np(g["W_w"]))
    assert_close(x, xr, torch.bfloat16, "x")
    assert_close(s, sr, torch.bfloat16, "s")


@pytest.mark.parametrize("T,n_r,d", [(300, 4, 256), (64, 4, 2560), (5, 2, 8), (33, 8, 4096)])
def test_gr_write_bit_exact(T, n_r, d):
    g = inputs.make_gr(T, n_r, d, 8, seed=7 * T + d)
    want_c, want_s = ogr.gr_write(_np(g["codes"]), _np(g["scales"]), _np(g["y"]), _np(g["s"]))
    codes, scales = g["codes"].cuda(), g["scales"].cuda()
    gdn.gdn_gr_write(codes, scales, g["y"].cuda(), g["s"].cuda())
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)


def test_gr_write_zero_output_and_zero_rows():
    g = inputs.make_gr(40, 4, 128, 8, seed=3)
    g["y"].zero_()
    g["codes"][5] = 0       # an all-zero token: every row of it stays zero, scale 1
    want_c, want_s = ogr.gr_write(_np(g["codes"]), _np(g["scales"]), _np(g["y"]), _np(g["s"]))
    codes, scales = g["codes"].cuda(), g["scales"].cuda()
    gdn.gdn_gr_write(codes, scales, g["y"].cuda(), g["s"].cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
    assert (want_s[5] == 1.0).all() and (want_c[5] == 0).all()


def test_gr_read_then_write_layer_step():
    """read -> (block output y) -> write, twice: the state the GPU carries
    equals the oracle's at every step (codes bit for bit, given the same s)."""
    g = inputs.make_gr(96, 4, 512, 64, seed=11)
    c = _cuda(g)
    codes, scales = c["codes"].clone(), c["scales"].clone()
    oc, osc = _np(g["codes"]), _np(g["scales"])
    for step in range(2):
        x, s = gdn.gdn_gr_read(codes, scales, c["gamma"], c["W_d"], c["W_u"], c["W_w"])
        xr, sr = ogr.gr_read(oc, osc, _np(g["gamma"]), _np(g["W_d"]), _np(g["W_u"]),
                             _np(g["W_w"]))
        assert_close(x, xr, torch.bfloat16, "x step %d" % step)
        # the write takes the same s on both sides (the oracle's, rounded to fp32)
        s_in = torch.tensor(sr, dtype=torch.float32)
        y = (x.float() * 0.5).to(torch.bfloat16)
        gdn.gdn_gr_write(codes, scales, y, s_in.cuda())
        oc, osc = ogr.gr_write(oc, osc, _np(y), s_in.numpy())
        torch.cuda.synchronize()
        np.testing.assert_array_equal(codes.cpu().numpy(), oc)
        np.testing.assert_array_equal(scales.cpu().numpy(), osc)


# (e, write scalar s as fp32 bits): with a zero state, y = (1, 3 2^(e-10), ...)
# and this s, the row's second value r = fl(s y) has r / scale just above an
# E4M3 rounding boundary while fp32 r * fl(1 / scale) falls on or below it.
_TIE_WRITES = [(-3, 1075015380), (-2, 1069550077), (-1, 1060131433), (0, 1072414671),
               (1, 1059623179), (2, 1059827673), (3, 1082118337), (4, 1080628333)]


def test_gr_write_rounds_the_exact_quotient():
    """Rows whose codes sit next to a rounding boundary: the kernel's codes
    are the rounding of the exact quotient r / scale, bit for bit."""
    T, n_r, d = len(_TIE_WRITES), 2, 32
    rng = np.random.default_rng(4)
    y = torch.tensor(rng.uniform(-0.9, 0.9, (T, d)), dtype=torch.float32).to(torch.bfloat16)
    s = torch.tensor(rng.uniform(0.5, 1.5, (T, n_r)), dtype=torch.float32)
    for t, (e, s_bits) in enumerate(_TIE_WRITES):
        y[t, 0] = 1.0
        y[t, 1] = 3 * 2.0 ** (e - 10)
        y[t, 2] = -3 * 2.0 ** (e - 10)
        s[t, 0] = float(np.array([s_bits], np.uint32).view(np.float32)[0])
    codes = torch.zeros((T, n_r, d), dtype=torch.uint8)
    scales = torch.ones((T, n_r), dtype=torch.float32)
    want_c, want_s = ogr.gr_write(codes.numpy(), scales.numpy(), _np(y), s.numpy())
    # the planted values do sit on the exact side of the boundary
    for t, (e, s_bits) in enumerate(_TIE_WRITES):
        sv = np.float32(s[t, 0].item())
        r = np.float32(sv * np.float32(3 * 2.0 ** (e - 10)))
        inv = np.float32(np.float32(1.0) / want_s[t, 0])
        recip = int(ogr.e4m3_encode(np.array([np.float32(r * inv)], np.float64))[0])
        assert int(want_c[t, 0, 1]) == recip + 1 and int(want_c[t, 0, 2]) == (recip + 1) | 0x80
    cd, sd = codes.cuda(), scales.cuda()
    gdn.gdn_gr_write(cd, sd, y.cuda(), s.cuda())
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    np.testing.assert_array_equal(cd.cpu().numpy(), want_c)
    np.testing.assert_array_equal(sd.cpu().numpy(), want_s)
