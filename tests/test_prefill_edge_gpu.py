"""Edge cases of the prefill kernels outside the workload recipes.

The tensor-core kernels run their MMAs on fp16 operands scaled by powers of
two chosen per chunk from block maxima; these cases push that scaling
(huge / tiny values, a large inverse), the decay (alpha ~ 0), repeated keys
(an ill-conditioned intra-chunk system), caller-normalised keys
(l2norm_qk = 0), a non-unit scale, the epilogue without a norm weight, and
an empty batch.  Each compares with the fp64 oracle; for scaled inputs the
absolute tolerance scales with the data.
"""
import numpy as np
import pytest
import torch

from gated_deltanet_scan_chunked_b200 import gdn, gdn_check_device_error, gdn_chunk_fwd, inputs
from tests._parity import assert_close, errors, oracle_prefill, to_device

pytestmark = pytest.mark.gpu

PATHS = ["simt", "tensor_single", "tensor_pair", "tensor_split"]


def _run(w, path, **kw):
    y, fs = gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, g=w.g, norm_w=w.norm_w,
                          initial_state=w.initial_state, cu_seqlens=w.cu_seqlens, path=path, **kw)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    return y, fs


def _check(got, ref, mag, what, rel=1e-2, abs_=2e-2):
    r, m = errors(got, ref)
    assert np.isfinite(r), "%s: non-finite output" % what
    assert r <= rel and m <= abs_ * mag, "%s: rel_l2=%.3e max_abs=%.3e (tol %.1e x %.3g)" % (
        what, r, m, abs_, mag)


def _case(T=200, seed=21, epilogue=True, s0_std=0.01):
    return inputs.make_prefill([T], 16, 48, 128, 128, seed=seed, epilogue=epilogue, s0_std=s0_std)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mag", [1e3, 1e-3])
def test_value_magnitudes(path, mag):
    """v and the initial state scaled by 1e3 / 1e-3: outputs without the
    epilogue scale along; nothing overflows or flushes to zero."""
    w = _case(epilogue=False)
    w.v = (w.v.float() * mag).to(torch.bfloat16)
    w.initial_state = w.initial_state * mag
    w = to_device(w)
    y, fs = _run(w, path)
    y_ref, s_ref, _ = oracle_prefill(w)
    _check(y, y_ref, mag, "y x%g %s" % (mag, path))
    _check(fs, s_ref, mag, "state x%g %s" % (mag, path))


@pytest.mark.parametrize("path", PATHS)
def test_strong_decay(path):
    """alpha ~ 7e-3 per token: decays underflow within a chunk."""
    w = _case()
    w.log_alpha = torch.full_like(w.log_alpha, -5.0)
    w = to_device(w)
    y, fs = _run(w, path)
    y_ref, s_ref, _ = oracle_prefill(w)
    _check(y, y_ref, 1.0, "y")
    _check(fs, s_ref, 1.0, "state")


@pytest.mark.parametrize("path", PATHS)
def test_no_decay_full_write(path):
    """alpha = 1, beta = 1: the delta rule alone (projections), no forgetting."""
    w = _case()
    w.log_alpha = torch.zeros_like(w.log_alpha)
    w.beta = torch.ones_like(w.beta)
    w = to_device(w)
    y, fs = _run(w, path)
    y_ref, s_ref, _ = oracle_prefill(w)
    _check(y, y_ref, 1.0, "y")
    _check(fs, s_ref, 1.0, "state")


@pytest.mark.parametrize("path", PATHS)
def test_repeated_keys(path):
    """The same key for every token with beta = 0.9, alpha = 1: the
    intra-chunk system I + A is as far from identity as unit keys allow."""
    w = _case(T=130)
    w.k = w.k[:1].expand_as(w.k).contiguous()
    w.beta = torch.full_like(w.beta, 0.9)
    w.log_alpha = torch.zeros_like(w.log_alpha)
    w = to_device(w)
    y, fs = _run(w, path)
    y_ref, s_ref, _ = oracle_prefill(w)
    _check(y, y_ref, 1.0, "y")
    _check(fs, s_ref, 1.0, "state")


@pytest.mark.parametrize("path", PATHS)
def test_caller_normalised_keys_and_scale(path):
    """l2norm_qk = 0 with unit-norm q/k from the caller, scale = 1/sqrt(d),
    epilogue gate without a norm weight."""
    w = _case()
    qn = w.q.float() / w.q.float().norm(dim=-1, keepdim=True)
    kn = w.k.float() / w.k.float().norm(dim=-1, keepdim=True)
    w.q = qn.to(torch.bfloat16)
    w.k = kn.to(torch.bfloat16)
    w.norm_w = None
    w = to_device(w)
    sc = 128 ** -0.5
    y, fs = _run(w, path, l2norm_qk=False, scale=sc)
    y_ref, s_ref, _ = oracle_prefill(w, l2norm=False, scale=sc)
    _check(y, y_ref, 1.0, "y")
    _check(fs, s_ref, 1.0, "state")


@pytest.mark.parametrize("path", ["auto", "simt", "tensor_split", "tensor_pair"])
def test_empty_batch(path):
    """total_T = 0: nothing to scan, the final state is the initial state."""
    w = to_device(_case(T=0))
    y, fs = _run(w, path)
    assert y.shape[0] == 0
    np.testing.assert_array_equal(fs.cpu().numpy(), w.initial_state.cpu().numpy())


def test_deterministic():
    """Two runs of the same inputs give bit-identical outputs (no atomics or
    order-dependent reductions on the data path)."""
    w = to_device(_case(T=300))
    y1, s1 = _run(w, "auto")
    y2, s2 = _run(w, "auto")
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


def test_bounded_wait_times_out_and_context_stays_usable():
    """A wait on a flag that nothing sets gives up, the host reads
    GDN_ERR_TIMEOUT once, and the next prefill still runs and is correct."""
    lib = gdn.load()
    assert lib.gdn_selftest_bounded_wait(1 << 12, None) == gdn.GDN_OK
    assert gdn_check_device_error() == gdn.GDN_ERR_TIMEOUT
    assert gdn_check_device_error() == gdn.GDN_OK  # cleared
    w = to_device(inputs.make_prefill([70], 2, 4, 16, 16, dtype=torch.float32, seed=3,
                                      epilogue=False))
    y, fs = gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, cu_seqlens=w.cu_seqlens)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    y_ref, s_ref, _ = oracle_prefill(w)
    assert_close(y, y_ref, torch.float32, "after timeout y")
