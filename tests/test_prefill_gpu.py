"""Chunked prefill on the GPU against the fp64 oracle.

Covers every kernel (``simt``: fp32 CUDA cores, every shape and dtype;
``tensor_single`` / ``tensor_pair`` / ``tensor_split``: the tcgen05 kernel for
bf16, d_k = d_v = 128, with one CTA, a cluster, or a chain CTA and two
preparation CTAs exchanging tiles through a global workspace per (sequence,
head)) on the workload recipes
(shortened where the oracle must see every output), ragged chunk tails,
empty and one-token sequences, packed batches, in-place state update,
split-and-carry, and sampled outputs at the full workload sizes.
"""
import numpy as np
import pytest
import torch

from gated_deltanet_scan_chunked_b200 import gdn, gdn_check_device_error, gdn_chunk_fwd, inputs
from tests._parity import assert_close, oracle_prefill, to_device

pytestmark = pytest.mark.gpu

BF16_PATHS = ["simt", "tensor_single", "tensor_pair", "tensor_split"]
# the split layout needs all 3 x items CTAs resident: batches of <= 49 items
MANY_ITEM_PATHS = ["simt", "tensor_single", "tensor_pair"]


def _run(w, path="auto", **kw):
    y, fs = gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, g=w.g, norm_w=w.norm_w,
                          initial_state=w.initial_state, cu_seqlens=w.cu_seqlens, path=path,
                          **kw)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    return y, fs


def _check_all(w, y, fs, dtype, what):
    y_ref, s_ref, _ = oracle_prefill(w)
    assert_close(y, y_ref, dtype, what + " y")
    assert_close(fs, s_ref, dtype, what + " final state")


def test_tiny_fp32():
    """The tiny oracle workload: T=64, 2 QK / 4 value heads, d=16, fp32."""
    w = to_device(inputs.workload("tiny"))
    y, fs = _run(w)
    _check_all(w, y, fs, torch.float32, "tiny")


@pytest.mark.parametrize("path", BF16_PATHS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200])
def test_model_shape_ragged_lengths(path, T):
    w = to_device(inputs.workload("prefill4k", T=T))
    y, fs = _run(w, path)
    _check_all(w, y, fs, torch.bfloat16, "T=%d %s" % (T, path))


@pytest.mark.parametrize("path", MANY_ITEM_PATHS)
@pytest.mark.parametrize("epilogue", [True, False])
def test_packed_varlen_small(path, epilogue):
    lengths = [0, 5, 64, 130, 1, 77, 0, 128]
    w = to_device(inputs.make_prefill(lengths, 16, 48, 128, 128, seed=7, epilogue=epilogue,
                                      s0_std=0.01))
    y, fs = _run(w, path)
    _check_all(w, y, fs, torch.bfloat16, "varlen %s" % path)
    # empty sequences: final state is the initial state
    np.testing.assert_array_equal(fs[0].cpu().numpy(), w.initial_state[0].cpu().numpy())


@pytest.mark.parametrize("epilogue", [True, False])
def test_one_cta_longest_first(epilogue):
    """More than 64 items with a workspace: the one-CTA layout takes the
    sequences longest first (the order is written into the workspace).  The
    results equal those of the in-order launch bit for bit and meet the bar
    against the oracle."""
    lengths = [0, 5, 64, 130, 1, 77, 0, 128, 300, 33]
    H_v = 8
    w = to_device(inputs.make_prefill(lengths, 2, H_v, 128, 128, seed=9, epilogue=epilogue,
                                      s0_std=0.01))
    nbytes = gdn.workspace_size(len(lengths), H_v, 128, 128)
    assert nbytes == 256
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    y1, fs1 = _run(w, "tensor_single", workspace=ws)
    y0, fs0 = _run(w, "tensor_single", workspace=None)
    torch.testing.assert_close(y1, y0, rtol=0, atol=0)
    torch.testing.assert_close(fs1, fs0, rtol=0, atol=0)
    order = ws[:4 * len(lengths)].view(torch.int32).cpu().tolist()
    assert order == sorted(range(len(lengths)), key=lambda s: (-lengths[s], s))
    _check_all(w, y1, fs1, torch.bfloat16, "longest first")


@pytest.mark.parametrize("path", ["tensor_split", "tensor_pair"])
@pytest.mark.parametrize("epilogue", [True, False])
def test_packed_varlen_few_heads(path, epilogue):
    """Packed sequences with 1 QK / 4 value heads (32 items): ragged, empty
    and one-token sequences through the small-batch layouts."""
    lengths = [0, 5, 64, 130, 1, 77, 0, 128]
    w = to_device(inputs.make_prefill(lengths, 1, 4, 128, 128, seed=8, epilogue=epilogue,
                                      s0_std=0.01))
    y, fs = _run(w, path)
    _check_all(w, y, fs, torch.bfloat16, "varlen few heads %s" % path)
    np.testing.assert_array_equal(fs[0].cpu().numpy(), w.initial_state[0].cpu().numpy())


def test_split_workspace_reuse_and_fallback():
    """One workspace serves consecutive calls (its flags are cleared by each
    call); without a workspace AUTO takes another layout, with the same
    results up to rounding."""
    w = to_device(inputs.make_prefill([333], 16, 48, 128, 128, seed=13, s0_std=0.01))
    ws = torch.empty(gdn.workspace_size(1, 48, 128, 128), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        outs.append(_run(w, "tensor_split", workspace=ws))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    y_nows, s_nows = _run(w, "auto", workspace=None)
    y_ref, s_ref, _ = oracle_prefill(w)
    assert_close(outs[0][0], y_ref, torch.bfloat16, "split y")
    assert_close(y_nows, y_ref, torch.bfloat16, "no-workspace y")
    assert_close(s_nows, s_ref, torch.bfloat16, "no-workspace state")


def test_split_rejects_batches_that_do_not_fit():
    w = to_device(inputs.make_prefill([10, 10], 16, 48, 128, 128, seed=1))  # 96 items
    with pytest.raises(gdn.GdnError) as e:
        _run(w, "tensor_split")
    assert e.value.status in (gdn.GDN_ERR_UNSUPPORTED, gdn.GDN_ERR_INVALID_ARG)


@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 128), (128, 16), (32, 64), (64, 32),
                                   (128, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_other_head_dims(dk, dv, dtype):
    w = to_device(inputs.make_prefill([100, 31], 2, 4, dk, dv, dtype=dtype, seed=dk + dv,
                                      s0_std=0.1))
    y, fs = _run(w, "simt")
    _check_all(w, y, fs, dtype, "d=%d/%d" % (dk, dv))


def test_fp32_model_shape():
    w = to_device(inputs.make_prefill([300], 16, 48, 128, 128, dtype=torch.float32, seed=3,
                                      s0_std=0.01))
    y, fs = _run(w)
    _check_all(w, y, fs, torch.float32, "fp32 d=128")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_in_place_state_update(path):
    # 2 sequences x 16 value heads: few enough items for every layout
    w = to_device(inputs.make_prefill([90, 40], 4, 16, 128, 128, seed=11, s0_std=0.01))
    y_ref, s_ref, _ = oracle_prefill(w)
    st = w.initial_state.clone()
    y, fs = gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, g=w.g, norm_w=w.norm_w,
                          initial_state=st, final_state=st, cu_seqlens=w.cu_seqlens, path=path)
    torch.cuda.synchronize()
    assert fs.data_ptr() == st.data_ptr()
    assert_close(st, s_ref, torch.bfloat16, "in-place state")
    assert_close(y, y_ref, torch.bfloat16, "in-place y")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_split_and_carry_equals_one_pass(path):
    w = to_device(inputs.make_prefill([333], 16, 48, 128, 128, seed=12, s0_std=0.01))
    y, fs = _run(w, path)
    t1 = 150
    a = dict(g=w.g[:t1], norm_w=w.norm_w, initial_state=w.initial_state, path=path)
    ya, fa = gdn_chunk_fwd(w.q[:t1], w.k[:t1], w.v[:t1], w.log_alpha[:t1], w.beta[:t1], **a)
    yb, fb = gdn_chunk_fwd(w.q[t1:], w.k[t1:], w.v[t1:], w.log_alpha[t1:], w.beta[t1:],
                           g=w.g[t1:], norm_w=w.norm_w, initial_state=fa, path=path)
    torch.cuda.synchronize()
    assert_close(torch.cat([ya, yb]), y.double().cpu().numpy(), torch.bfloat16, "split y")
    assert_close(fb, fs.cpu().numpy(), torch.bfloat16, "split state")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_model_shape_full_T4096(path):
    """The model-shape workload at full size; the oracle checks every output."""
    w = to_device(inputs.workload("prefill4k"))
    y, fs = _run(w, path)
    _check_all(w, y, fs, torch.bfloat16, "T=4096 %s" % path)


@pytest.mark.parametrize("path", BF16_PATHS)
def test_native_context_T262144_sampled_heads(path):
    """T = 262,144 with a random initial state; the oracle recomputes two value
    heads (from different QK heads) over the whole sequence."""
    w = inputs.workload("prefill256k", device="cuda")
    y, fs = _run(w, path)
    heads = [5, 40]
    y_ref, s_ref, _ = oracle_prefill(w, heads=heads, n_threads=len(heads))
    assert_close(y[:, heads], y_ref, torch.bfloat16, "y")
    assert_close(fs[:, heads], s_ref, torch.bfloat16, "final state")


@pytest.mark.parametrize("path", MANY_ITEM_PATHS)
def test_packed_varlen_full_sampled(path):
    """24 sequences (~200k tokens) with their own states; sampled
    (sequence, head) pairs against the oracle, plus no leakage: every final
    state differs from its initial state and from its neighbours'."""
    w = inputs.workload("varlen", device="cuda")
    y, fs = _run(w, path)
    cu = w.cu_seqlens.cpu().numpy()
    seqs, heads = [0, 11, 23], [0, 17, 47]
    y_ref, s_ref, tok = oracle_prefill(w, heads=heads, seqs=seqs, n_threads=9)
    tok_t = torch.as_tensor(tok, device="cuda")
    assert_close(y[tok_t][:, heads], y_ref, torch.bfloat16, "y")
    assert_close(fs[seqs][:, heads], s_ref, torch.bfloat16, "final state")
    assert len(cu) == 25


def test_malformed_cu_seqlens_reported_by_device():
    """A non-monotone cu_seqlens cannot be checked on the host without a sync;
    the kernel skips the bad sequences and flags the error word."""
    w = to_device(inputs.make_prefill([10, 10, 10], 2, 4, 16, 16, dtype=torch.float32, seed=1))
    bad = torch.tensor([0, 15, 12, 30], dtype=torch.int32, device="cuda")
    gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, cu_seqlens=bad)
    assert gdn_check_device_error() == gdn.GDN_ERR_INVALID_ARG
    assert gdn_check_device_error() == gdn.GDN_OK  # cleared
