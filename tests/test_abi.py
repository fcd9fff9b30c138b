"""CPU-side checks of the C ABI: the library loads without a GPU, exports
every function include/gdn.h declares, and rejects bad arguments on the
host before touching the device."""
import ctypes

import pytest

from gated_deltanet_scan_chunked_b200 import build as gbuild
from gated_deltanet_scan_chunked_b200 import gdn


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gdn.load()


def test_exports_every_declared_function(lib):
    names = gdn.header_functions()
    assert set(names) >= {"gdn_chunk_fwd", "gdn_chunk_fwd_path", "gdn_chunk_fwd_ws", "gdn_chunk_bwd",
                          "gdn_chunk_bwd_workspace_size",
                          "gdn_chunk_fwd_workspace_size", "gdn_decode_step",
                          "gdn_check_device_error", "gdn_status_string", "gdn_version"}
    for n in names:
        assert hasattr(lib, n), "libgdn.so does not export %s" % n


def test_status_strings_and_version(lib):
    assert gdn.status_string(0) == "ok"
    assert "timed out" in gdn.status_string(4)
    assert gdn.status_string(99) == "unknown status"
    assert lib.gdn_version() >= 100


FAKE = 0x1000  # a 16-byte aligned non-null address; never dereferenced


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, g=None, w=None, s0=None, cu=None,
             n_seq=1, T=64, Hqk=16, Hv=48, dk=128, dv=128, dt=0, l2=1, e1=1e-6, e2=1e-6,
             sc=1.0, y=FAKE, fs=None, path=0)
    a.update(kw)
    return lib.gdn_chunk_fwd_path(a["q"], a["k"], a["v"], a["la"], a["b"], a["g"], a["w"],
                                  a["s0"], a["cu"], a["n_seq"], a["T"], a["Hqk"], a["Hv"],
                                  a["dk"], a["dv"], a["dt"], a["l2"], a["e1"], a["e2"],
                                  a["sc"], a["y"], a["fs"], a["path"], None)


def _decode(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, g=None, w=None, s=FAKE, N=4, Hqk=16,
             Hv=48, dk=128, dv=128, dt=0, l2=1, e1=1e-6, e2=1e-6, sc=1.0, y=FAKE)
    a.update(kw)
    return lib.gdn_decode_step(a["q"], a["k"], a["v"], a["la"], a["b"], a["g"], a["w"],
                               a["s"], a["N"], a["Hqk"], a["Hv"], a["dk"], a["dv"], a["dt"],
                               a["l2"], a["e1"], a["e2"], a["sc"], a["y"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(y=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hv=40), gdn.GDN_ERR_INVALID_ARG),          # 40 % 16 != 0
    (dict(Hqk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(n_seq=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(n_seq=2), gdn.GDN_ERR_INVALID_ARG),        # several sequences need cu_seqlens
    (dict(T=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dt=7), gdn.GDN_ERR_UNSUPPORTED),
    (dict(e1=-1.0), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=FAKE + 8), gdn.GDN_ERR_INVALID_ARG),     # misaligned
    (dict(cu=FAKE + 2, n_seq=2), gdn.GDN_ERR_INVALID_ARG),
    (dict(path=9), gdn.GDN_ERR_INVALID_ARG),
    (dict(s0=FAKE, fs=FAKE + 4096), gdn.GDN_ERR_INVALID_ARG),  # partial overlap
])
def test_chunk_fwd_rejects_bad_arguments_on_host(lib, kw, code):
    assert _chunk(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(s=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hv=17), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=8), gdn.GDN_ERR_UNSUPPORTED),
    (dict(y=FAKE + 4), gdn.GDN_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments_on_host(lib, kw, code):
    assert _decode(lib, **kw) == code


def _chunk_ws(lib, ws=None, ws_bytes=0, path=0, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, g=None, w=None, s0=None, cu=None,
             n_seq=1, T=64, Hqk=16, Hv=48, dk=128, dv=128, dt=0, l2=1, e1=1e-6, e2=1e-6,
             sc=1.0, y=FAKE, fs=None)
    a.update(kw)
    return lib.gdn_chunk_fwd_ws(a["q"], a["k"], a["v"], a["la"], a["b"], a["g"], a["w"],
                                a["s0"], a["cu"], a["n_seq"], a["T"], a["Hqk"], a["Hv"],
                                a["dk"], a["dv"], a["dt"], a["l2"], a["e1"], a["e2"],
                                a["sc"], a["y"], a["fs"], path, ws, ws_bytes, None)


def test_workspace_size(lib):
    """Scan layout: 128 bytes of flags per item (padded to 256), then eight
    90,368-byte hand-off slots per item; beyond 64 items, the one-CTA
    layout's sequence order (n_seq int32, padded to 256) up to 1024
    sequences; nothing for shapes the tensor-core kernel cannot serve."""
    one = 8 * 73984
    assert gdn.workspace_size(1, 48, 128, 128) == 48 * 128 + 48 * one
    assert gdn.workspace_size(1, 1, 128, 128) == 256 + one
    assert gdn.workspace_size(2, 32, 128, 128) == 64 * 128 + 64 * one
    assert gdn.workspace_size(3, 32, 128, 128) == 256        # more than 64 items: the order
    assert gdn.workspace_size(24, 48, 128, 128) == 256
    assert gdn.workspace_size(100, 48, 128, 128) == 512
    assert gdn.workspace_size(1024, 48, 128, 128) == 4096
    assert gdn.workspace_size(1025, 48, 128, 128) == 0
    assert gdn.workspace_size(1, 48, 64, 128) == 0
    assert gdn.workspace_size(1, 48, 128, 128, dtype=__import__("torch").float32) == 0
    assert lib.gdn_chunk_fwd_workspace_size(0, 48, 128, 128, 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(ws=FAKE + 16, ws_bytes=1 << 30), gdn.GDN_ERR_INVALID_ARG),   # not 256-aligned
    (dict(ws=FAKE, ws_bytes=1000), gdn.GDN_ERR_INVALID_ARG),           # too small
    (dict(path=5), gdn.GDN_ERR_INVALID_ARG),                           # split, no workspace
    (dict(path=5, ws=FAKE, ws_bytes=1 << 30, dk=64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(path=5, ws=FAKE, ws_bytes=1 << 30, dt=1), gdn.GDN_ERR_UNSUPPORTED),
    (dict(path=6), gdn.GDN_ERR_INVALID_ARG),
])
def test_chunk_fwd_ws_rejects_bad_workspace_on_host(lib, kw, code):
    assert _chunk_ws(lib, **kw) == code


def test_decode_with_no_sequences_is_a_no_op(lib):
    assert _decode(lib, N=0, q=None, s=None, y=None) == gdn.GDN_OK


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(4, 1, 16)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_fwd(q, q, torch.zeros(4, 1, 16), torch.zeros(4, 1), torch.zeros(4, 1))


def test_static_workspace_call_rejects_on_host(lib):
    """gdn_chunk_fwd_static_ws: over-capacity batches (96 items) and shapes
    the split layout does not serve are refused before any CUDA call."""
    def call(**kw):
        a = dict(cu=FAKE, n_seq=2, Hv=48, dk=128, dt=0)
        a.update(kw)
        return lib.gdn_chunk_fwd_static_ws(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                                           a["cu"], a["n_seq"], 64, 16, a["Hv"], a["dk"], 128,
                                           a["dt"], 1, 1e-6, 1e-6, 1.0, FAKE, None, None)
    assert call() == gdn.GDN_ERR_UNSUPPORTED
    assert call(n_seq=1, cu=None, dk=64) == gdn.GDN_ERR_UNSUPPORTED
    assert call(n_seq=1, cu=None, dt=1) == gdn.GDN_ERR_UNSUPPORTED
    assert call(n_seq=0) == gdn.GDN_ERR_INVALID_ARG
    # argument errors come first, with the codes gdn_chunk_fwd_ws gives
    for kw in (dict(n_seq=1, cu=None, dk=0), dict(n_seq=1, cu=None, Hv=47),
               dict(n_seq=1, cu=None, dt=7), dict(n_seq=1, cu=None, dk=-128)):
        a = dict(cu=FAKE, n_seq=2, Hv=48, dk=128, dt=0)
        a.update(kw)
        ref = lib.gdn_chunk_fwd_ws(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, a["cu"],
                                   a["n_seq"], 64, 16, a["Hv"], a["dk"], 128, a["dt"], 1, 1e-6,
                                   1e-6, 1.0, FAKE, None, 0, None, 0, None)
        assert ref in (gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED)
        assert call(**kw) == ref, kw
    assert call(n_seq=1, cu=None, dk=0) == gdn.GDN_ERR_INVALID_ARG


def _multi(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, g=None, w=None, si=FAKE, so=FAKE,
             sn=None, N=4, T=4, Hqk=16, Hv=48, dk=128, dv=128, dt=0, y=FAKE)
    a.update(kw)
    return lib.gdn_decode_multi(a["q"], a["k"], a["v"], a["la"], a["b"], a["g"], a["w"],
                                a["si"], a["so"], a["sn"], a["N"], a["T"], a["Hqk"], a["Hv"],
                                a["dk"], a["dv"], a["dt"], 1, 1e-6, 1e-6, 1.0, a["y"], None)


STATE_BYTES = 4 * 48 * 128 * 128 * 4


@pytest.mark.parametrize("kw,code", [
    (dict(T=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(si=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(so=FAKE + 4096), gdn.GDN_ERR_INVALID_ARG),                   # partial overlap
    (dict(so=FAKE + STATE_BYTES, sn=FAKE + 4096), gdn.GDN_ERR_INVALID_ARG),  # snapshots overlap
    (dict(sn=FAKE + 8), gdn.GDN_ERR_INVALID_ARG),                      # misaligned
    (dict(dk=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(T=33), gdn.GDN_ERR_UNSUPPORTED),                             # over 32 tokens
    (dict(T=0, q=None), gdn.GDN_OK),                                   # no-op
    (dict(N=0, y=None), gdn.GDN_OK),
])
def test_decode_multi_rejects_bad_arguments_on_host(lib, kw, code):
    assert _multi(lib, **kw) == code


def _bwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, g=None, w=None, s0=None, cu=None,
             n_seq=1, T=64, Hqk=16, Hv=48, dk=128, dv=128, dt=0, dy=FAKE, dsT=None,
             dq=FAKE, dkk=FAKE, dvv=FAKE, dla=FAKE, db=FAKE, dg=None, dw=None, ds0=None,
             ws=FAKE, wsb=1 << 40)
    a.update(kw)
    return lib.gdn_chunk_bwd(a["q"], a["k"], a["v"], a["la"], a["b"], a["g"], a["w"], a["s0"],
                             a["cu"], a["n_seq"], a["T"], a["Hqk"], a["Hv"], a["dk"], a["dv"],
                             a["dt"], 1, 1e-6, 1e-6, 1.0, a["dy"], a["dsT"], a["dq"], a["dkk"],
                             a["dvv"], a["dla"], a["db"], a["dg"], a["dw"], a["ds0"], a["ws"],
                             a["wsb"], None)


def test_bwd_workspace_size(lib):
    """Backward workspace: grows with chunks x heads; 0 for unsupported dims."""
    n1 = gdn.bwd_workspace_size(1, 4096, 16, 48, 128, 128)
    assert 1.3e9 < n1 < 1.6e9
    assert gdn.bwd_workspace_size(1, 8192, 16, 48, 128, 128) > 1.9 * n1
    assert gdn.bwd_workspace_size(1, 64, 16, 48, 96, 128) == 0
    assert gdn.bwd_workspace_size(1, 64, 16, 40, 128, 128) == 0
    assert gdn.bwd_workspace_size(0, 64, 16, 48, 128, 128) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), gdn.GDN_ERR_INVALID_ARG),                       # no workspace
    (dict(ws=FAKE + 16), gdn.GDN_ERR_INVALID_ARG),                  # not 256-aligned
    (dict(wsb=1000), gdn.GDN_ERR_INVALID_ARG),                      # too small
    (dict(dy=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dq=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(g=FAKE), gdn.GDN_ERR_INVALID_ARG),                        # g without dg
    (dict(dg=FAKE), gdn.GDN_ERR_INVALID_ARG),                       # dg without g
    (dict(dw=FAKE), gdn.GDN_ERR_INVALID_ARG),                       # dnorm_w without g
    (dict(dvv=FAKE + 4), gdn.GDN_ERR_INVALID_ARG),                  # misaligned
    (dict(dk=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dt=3), gdn.GDN_ERR_UNSUPPORTED),
    (dict(n_seq=2), gdn.GDN_ERR_INVALID_ARG),                       # needs cu_seqlens
    (dict(Hv=40), gdn.GDN_ERR_INVALID_ARG),
])
def test_chunk_bwd_rejects_bad_arguments_on_host(lib, kw, code):
    assert _bwd(lib, **kw) == code


def test_conv_entry_points_reject_on_host(lib):
    """Front-end calls: overlapping conv states, missing weights, outputs on
    top of inputs, a missing or short workspace are refused on the host."""
    C4 = (2 * 16 * 128 + 48 * 128) * 16  # bytes of conv_w
    ns = 2 * 48 * 3 * 384 * 4            # bytes of a 2-sequence conv state

    def fe(**kw):
        a = dict(q=FAKE, k=FAKE + (1 << 24), v=FAKE + (2 << 24), w=FAKE + (3 << 24), si=None,
                 so=None, cu=FAKE + (4 << 24), n_seq=2, T=64, dk=128, qo=FAKE + (5 << 24),
                 ko=FAKE + (6 << 24), vo=FAKE + (7 << 24))
        a.update(kw)
        return lib.gdn_conv_frontend(a["q"], a["k"], a["v"], a["w"], a["si"], a["so"], a["cu"],
                                     a["n_seq"], a["T"], 16, 48, a["dk"], 128, 0, a["qo"],
                                     a["ko"], a["vo"], None)
    S = FAKE + (8 << 24)
    assert fe(w=None) == gdn.GDN_ERR_INVALID_ARG
    assert fe(si=S, so=S) == gdn.GDN_ERR_INVALID_ARG              # in place is refused
    assert fe(si=S, so=S + ns - 256) == gdn.GDN_ERR_INVALID_ARG   # partial overlap
    assert fe(qo=FAKE) == gdn.GDN_ERR_INVALID_ARG                 # output on its input
    assert fe(vo=FAKE + (1 << 24) + 64) == gdn.GDN_ERR_INVALID_ARG  # output inside k
    assert fe(dk=96) == gdn.GDN_ERR_UNSUPPORTED
    assert C4 > 0

    n = gdn.conv_workspace_size(2, 64, 16, 48, 128, 128)
    assert n >= 64 * (2 * 16 * 128 + 48 * 128) * 2
    assert gdn.conv_workspace_size(2, 64, 16, 48, 96, 128) == 0

    def cf(ws, wsb):
        return lib.gdn_chunk_fwd_conv(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, None, None,
                                      None, FAKE, 2, 64, 16, 48, 128, 128, 0, 1, 1e-6, 1e-6,
                                      1.0, FAKE, None, 0, ws, wsb, None)
    assert cf(None, 0) == gdn.GDN_ERR_INVALID_ARG
    assert cf(S, n - 256) == gdn.GDN_ERR_INVALID_ARG
    assert cf(S + 16, n) == gdn.GDN_ERR_INVALID_ARG

    def dc(**kw):
        a = dict(w=FAKE, cs=S, si=FAKE + (9 << 24), so=FAKE + (9 << 24), sn=None)
        a.update(kw)
        return lib.gdn_decode_conv(FAKE, FAKE, FAKE, a["w"], a["cs"], FAKE, FAKE, None, None,
                                   a["si"], a["so"], a["sn"], 4, 2, 16, 48, 128, 128, 0, 1,
                                   1e-6, 1e-6, 1.0, FAKE, None)
    assert dc(w=None) == gdn.GDN_ERR_INVALID_ARG
    assert dc(cs=FAKE + (9 << 24) + 4096) == gdn.GDN_ERR_INVALID_ARG  # inside the state
    assert dc(cs=S + 8) == gdn.GDN_ERR_INVALID_ARG                     # misaligned


def test_gr_entry_points_reject_on_host(lib):
    n = gdn.gr_read_workspace_size(64, 4, 2560, 320)
    assert n > 64 * 4 * 2560 * 2 * 2
    assert gdn.gr_read_workspace_size(64, 9, 2560, 320) == 0      # more than 8 branches
    assert gdn.gr_read_workspace_size(64, 4, 2561, 320) == 0      # d not a multiple of 8
    assert gdn.gr_read_workspace_size(64, 4, 2560, 12) == 0       # rank not a multiple of 8

    def rd(**kw):
        a = dict(c=FAKE, ws=FAKE, wsb=n, T=64, nr=4, d=2560, r=320, x=FAKE, s=FAKE)
        a.update(kw)
        return lib.gdn_gr_read(a["c"], FAKE, FAKE, FAKE, FAKE, FAKE, a["T"], a["nr"], a["d"],
                               a["r"], 1e-6, a["x"], a["s"], a["ws"], a["wsb"], None)
    assert rd(ws=None) == gdn.GDN_ERR_INVALID_ARG
    assert rd(wsb=n - 256) == gdn.GDN_ERR_INVALID_ARG
    assert rd(c=None) == gdn.GDN_ERR_INVALID_ARG
    assert rd(nr=0) == gdn.GDN_ERR_INVALID_ARG
    assert rd(x=FAKE + 8) == gdn.GDN_ERR_INVALID_ARG
    assert rd(T=0, c=None, x=None, s=None, wsb=gdn.gr_read_workspace_size(0, 4, 2560, 320)) \
        == gdn.GDN_OK
    assert lib.gdn_gr_write(FAKE, FAKE, FAKE, FAKE, 64, 4, 12, None) == gdn.GDN_ERR_INVALID_ARG
    assert lib.gdn_gr_write(None, FAKE, FAKE, FAKE, 64, 4, 16, None) == gdn.GDN_ERR_INVALID_ARG
    assert lib.gdn_gr_write(None, None, None, None, 0, 4, 16, None) == gdn.GDN_OK


def test_selftest_rejects_nonpositive_iterations(lib):
    assert lib.gdn_selftest_bounded_wait(0, None) == gdn.GDN_ERR_INVALID_ARG
