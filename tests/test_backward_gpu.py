"""Backward of the chunked scan on the GPU against the oracle's fp64 adjoint.

The CUDA backward (gdn_chunk_bwd: chunkwise, fp32 on CUDA cores) is compared
gradient by gradient with ``oracle.backward`` on the same seeded inputs: every
output at sizes the oracle finishes in seconds (ragged chunk tails, empty and
one-token sequences, packed batches, every supported head dimension, with and
without the epilogue and the L2 norm), and one QK group of heads at the
model shape T = 4,096.

Bar: relative L2 error <= 1e-4 per gradient tensor (the fp32 parity bar;
the backward computes in fp32 whatever the input dtype, from inputs the
oracle sees rounded identically).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_scan_chunked_b200 import gdn, gdn_check_device_error, gdn_chunk_bwd, inputs
from tests._parity import errors, to_device

pytestmark = pytest.mark.gpu

REL = 1e-4
NAMES = ["dq", "dk", "dv", "dlog_alpha", "dbeta", "d_initial_state", "dg", "dnorm_w"]


def _cpu(x):
    return None if x is None else x.detach().to("cpu", torch.float32)


def _oracle(w, dy, dsT, heads=None, **kw):
    """oracle.backward on the value heads ``heads`` (all when None); heads
    must be whole QK groups so that dq, dk are complete."""
    Hqk, Hv = w.q.shape[1], w.v.shape[1]
    G = Hv // Hqk
    hv = list(range(Hv)) if heads is None else list(heads)
    hq = sorted(set(h // G for h in hv))
    pick = lambda x, idx: None if x is None else _cpu(x)[:, idx]
    s0 = None if w.initial_state is None else _cpu(w.initial_state)[:, hv]
    ds = None if dsT is None else _cpu(dsT)[:, hv]
    return oracle.backward(pick(w.q, hq), pick(w.k, hq), pick(w.v, hv),
                           pick(w.log_alpha, hv), pick(w.beta, hv), pick(dy, hv),
                           g=pick(w.g, hv), norm_w=_cpu(w.norm_w), initial_state=s0,
                           d_final_state=ds, cu_seqlens=_cpu(w.cu_seqlens).to(torch.int64),
                           **kw), hv, hq


def _gpu(w, dy, dsT, **kw):
    out = gdn_chunk_bwd(w.q, w.k, w.v, w.log_alpha, w.beta, dy, g=w.g, norm_w=w.norm_w,
                        initial_state=w.initial_state, d_final_state=dsT,
                        cu_seqlens=w.cu_seqlens, **kw)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    return out


def _compare(got, ref, hv=None, hq=None, what=""):
    for n in NAMES:
        if n not in ref:
            continue
        g = got[n].detach().cpu().double().numpy()
        if hv is not None and n in ("dv", "dlog_alpha", "dbeta", "dg"):
            g = g[:, hv]
        if hv is not None and n in ("dq", "dk"):
            g = g[:, hq]
        if hv is not None and n == "d_initial_state":
            g = g[:, hv]
        rel, mx = errors(g, ref[n])
        assert rel <= REL, "%s %s: rel_l2=%.3e (bar %.0e) max_abs=%.3e" % (what, n, rel, REL, mx)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("epilogue", [True, False])
def test_packed_batch_model_dims(dtype, epilogue):
    lengths = [130, 0, 77, 64, 1]
    w = to_device(inputs.make_prefill(lengths, 2, 4, 128, 128, dtype=dtype, seed=11,
                                      epilogue=epilogue, s0_std=0.1))
    dy, dsT = inputs.make_cotangents(w, seed=11)
    got = _gpu(w, dy, dsT)
    ref, _, _ = _oracle(w, dy, dsT)
    _compare(got, ref, what="bf16" if dtype == torch.bfloat16 else "fp32")


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 16)])
def test_head_dims_without_l2norm(dk, dv):
    lengths = [100, 3]
    w = inputs.make_prefill(lengths, 1, 2, dk, dv, dtype=torch.float32, seed=dk + dv,
                            epilogue=True, s0_std=0.1)
    # without the in-kernel norm the caller supplies unit-scale keys
    w.q.div_(dk ** 0.5)
    w.k.div_(dk ** 0.5)
    w = to_device(w)
    dy, dsT = inputs.make_cotangents(w, seed=5)
    got = _gpu(w, dy, dsT, l2norm_qk=False, scale=0.5)
    ref, _, _ = _oracle(w, dy, dsT, l2norm=False, scale=0.5)
    _compare(got, ref, what="dk=%d dv=%d" % (dk, dv))


def test_no_final_gradient_no_initial_state():
    w = to_device(inputs.make_prefill([200], 1, 3, 64, 64, seed=3, epilogue=False))
    dy, _ = inputs.make_cotangents(w, seed=3, final_grad=False)
    got = _gpu(w, dy, None)
    ref, _, _ = _oracle(w, dy, None)
    _compare(got, ref, what="no dS_T")


def test_only_final_gradient():
    """dy = 0: every gradient comes through the final state alone."""
    w = to_device(inputs.make_prefill([90], 1, 2, 32, 32, dtype=torch.float32, seed=4,
                                      epilogue=False, s0_std=0.2))
    dy, dsT = inputs.make_cotangents(w, seed=4)
    dy.zero_()
    got = _gpu(w, dy, dsT)
    ref, _, _ = _oracle(w, dy, dsT)
    _compare(got, ref, what="dy=0")


def test_empty_batch_passes_final_gradient_through():
    w = to_device(inputs.make_prefill([0, 0], 1, 2, 16, 16, dtype=torch.float32, seed=1,
                                      epilogue=False, s0_std=0.1))
    dy, dsT = inputs.make_cotangents(w, seed=1)
    got = _gpu(w, dy, dsT)
    assert torch.equal(got["d_initial_state"], dsT)


def test_workspace_reuse_and_rejects():
    w = to_device(inputs.make_prefill([70, 10], 1, 2, 32, 32, seed=2, epilogue=True))
    dy, dsT = inputs.make_cotangents(w, seed=2)
    n = gdn.bwd_workspace_size(2, 80, 1, 2, 32, 32)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    a = _gpu(w, dy, dsT, workspace=ws)
    ws.fill_(0xff)  # stale contents must not matter
    b = _gpu(w, dy, dsT, workspace=ws)
    for k_ in a:
        assert torch.equal(a[k_], b[k_]), k_
    with pytest.raises(gdn.GdnError):
        _gpu(w, dy, dsT, workspace=ws[: n - 256])


def test_model_shape_one_group_sampled():
    """T = 4,096 with the model's 16 / 48 heads: the whole launch, checked on
    the three value heads of QK head 5 (dq, dk of that QK head complete)."""
    w = to_device(inputs.workload("prefill4k"))
    dy, dsT = inputs.make_cotangents(w, seed=4096)
    got = _gpu(w, dy, dsT)
    ref, hv, hq = _oracle(w, dy, dsT, heads=[15, 16, 17])
    ref.pop("dnorm_w")  # needs every head
    _compare(got, ref, hv, hq, what="T=4096")


def test_ungrouped_heads_fp32():
    """H_qk = H_v (one value head per QK head) with a ragged packed batch."""
    w = to_device(inputs.make_prefill([65, 3], 2, 2, 32, 16, dtype=torch.float32, seed=13,
                                      epilogue=True, s0_std=0.1))
    dy, dsT = inputs.make_cotangents(w, seed=13)
    got = _gpu(w, dy, dsT)
    ref, _, _ = _oracle(w, dy, dsT)
    _compare(got, ref, what="H_qk = H_v")


def test_long_sequence_one_group_sampled():
    """T = 16,384 (256 chunks per head) with an initial state: the whole launch
    at the model's head counts, checked on the value heads of QK head 10."""
    w = inputs.workload("prefill256k", T=16384, device="cuda")
    dy, dsT = inputs.make_cotangents(w, seed=16384)
    got = _gpu(w, dy, dsT)
    ref, hv, hq = _oracle(w, dy, dsT, heads=[30, 31, 32])
    ref.pop("dnorm_w")
    _compare(got, ref, hv, hq, what="T=16384")
