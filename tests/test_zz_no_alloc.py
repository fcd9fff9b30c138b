"""gdn_chunk_fwd_static_ws: the split-layout prefill with the library's own
fixed workspace.  Collected last (file name), so it runs both alone and after
every other test of the session; it must give the same bits as the
caller-workspace entry point on two consecutive calls (the static array's
flags are cleared by every call, so a second call cannot see the first's)."""
import pytest
import torch

from gated_deltanet_scan_chunked_b200 import gdn, inputs
from tests._parity import assert_close, oracle_prefill, to_device

pytestmark = pytest.mark.gpu


def _args(w):
    return (w.q, w.k, w.v, w.log_alpha, w.beta)


def _kw(w):
    return dict(g=w.g, norm_w=w.norm_w, initial_state=w.initial_state, cu_seqlens=w.cu_seqlens)


def test_static_workspace_matches_caller_workspace_twice():
    w = to_device(inputs.make_prefill([333], 16, 48, 128, 128, seed=31, s0_std=0.01))
    ws = torch.empty(gdn.workspace_size(1, 48, 128, 128), dtype=torch.uint8, device="cuda")
    y_ref, s_ref = gdn.gdn_chunk_fwd(*_args(w), **_kw(w), path="tensor_split", workspace=ws)
    # outputs allocated up front, so that the device's free memory can show
    # that the calls themselves allocate nothing
    y = torch.empty_like(y_ref)
    fs = torch.empty_like(s_ref)
    gdn.gdn_chunk_fwd_static_ws(*_args(w), **_kw(w), y=y, final_state=fs)  # first call: set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        y.zero_()
        fs.zero_()
        gdn.gdn_chunk_fwd_static_ws(*_args(w), **_kw(w), y=y, final_state=fs)
        torch.cuda.synchronize()
        assert gdn.gdn_check_device_error() == gdn.GDN_OK
        assert torch.equal(y, y_ref) and torch.equal(fs, s_ref)
    assert torch.cuda.mem_get_info()[0] == free0
    y_o, s_o, _ = oracle_prefill(w)
    assert_close(y, y_o, torch.bfloat16, "static-workspace y")
    assert_close(fs, s_o, torch.bfloat16, "static-workspace state")


def test_static_workspace_packed_batch_twice():
    """8 packed sequences x 4 value heads (32 items) with ragged / empty
    sequences, against the caller-workspace call, twice in a row."""
    w = to_device(inputs.make_prefill([0, 5, 64, 130, 1, 77, 0, 128], 1, 4, 128, 128, seed=32,
                                      s0_std=0.01))
    ref = gdn.gdn_chunk_fwd(*_args(w), **_kw(w), path="tensor_split")
    for _ in range(2):
        out = gdn.gdn_chunk_fwd_static_ws(*_args(w), **_kw(w))
        torch.cuda.synchronize()
        assert gdn.gdn_check_device_error() == gdn.GDN_OK
        assert torch.equal(out[0], ref[0]) and torch.equal(out[1], ref[1])


def test_static_workspace_rejects_oversize_batch():
    w = to_device(inputs.make_prefill([10, 10], 16, 48, 128, 128, seed=33))  # 96 items
    with pytest.raises(gdn.GdnError) as e:
        gdn.gdn_chunk_fwd_static_ws(*_args(w), **_kw(w))
    assert e.value.status == gdn.GDN_ERR_UNSUPPORTED
