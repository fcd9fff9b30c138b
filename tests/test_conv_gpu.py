"""The front end (short depthwise causal conv of kernel 4 + SiLU) on the GPU
against the oracle: the standalone kernel (gdn_conv_frontend), the prefill
on pre-conv inputs (gdn_chunk_fwd_conv) on every path, and the decode with
the front end fused (gdn_decode_conv), including a decode that continues a
prefill.  Carried conv states are compared bit for bit (they are copies of
inputs); outputs within the library's tolerances.

On the tensor-core path gdn_chunk_fwd_conv hands the front end's outputs to
the scan in the input dtype, as the scan's q/k/v inputs are in that dtype;
its oracle then rounds the oracle's own conv outputs to that dtype (on the
host) before the recurrence.  The portable prefill kernel and the decode take
the front end fused, keep the activations in fp32, and are compared with the
unrounded oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_scan_chunked_b200 import (gdn, gdn_check_device_error, gdn_chunk_fwd_conv,
                                              gdn_conv_frontend, gdn_decode_conv, inputs)
from tests._parity import assert_close, errors, to_device

pytestmark = pytest.mark.gpu


def _np(x):
    return None if x is None else x.detach().to("cpu", torch.float64).numpy()


def _mixed(q, k, v):
    T = q.shape[0]
    return np.concatenate([_np(q).reshape(T, -1), _np(k).reshape(T, -1), _np(v).reshape(T, -1)], 1)


def _to_oracle_state(st, H_qk, d_k, d_v):
    """[n, H_v, 3, 2 d_k + d_v] per value head -> [n, 3, C] over all channels."""
    if st is None:
        return None
    st = _np(st)
    n, Hv = st.shape[:2]
    G = Hv // H_qk
    q = st[:, ::G, :, :d_k].transpose(0, 2, 1, 3).reshape(n, 3, -1)
    k = st[:, ::G, :, d_k:2 * d_k].transpose(0, 2, 1, 3).reshape(n, 3, -1)
    v = st[:, :, :, 2 * d_k:].transpose(0, 2, 1, 3).reshape(n, 3, -1)
    return np.concatenate([q, k, v], 2)


def _oracle_conv(q, k, v, w, st_in, cu):
    H_qk, d_k = q.shape[1], q.shape[2]
    d_v = v.shape[2]
    y, so = oracle.conv(_mixed(q, k, v).astype(np.float32), _np(w).astype(np.float32),
                        None if st_in is None else
                        _to_oracle_state(st_in, H_qk, d_k, d_v).astype(np.float32),
                        cu_seqlens=_np(cu).astype(np.int64))
    T = q.shape[0]
    nq = H_qk * d_k
    qo = y[:, :nq].reshape(T, H_qk, d_k)
    ko = y[:, nq:2 * nq].reshape(T, H_qk, d_k)
    vo = y[:, 2 * nq:].reshape(T, v.shape[1], d_v)
    return qo, ko, vo, so


def _check_state(got, want_oracle_layout, H_qk, d_k, d_v):
    g = _np(got)
    G = g.shape[1] // H_qk
    # every copy of a group's q/k part is written
    for m in range(G):
        np.testing.assert_array_equal(g[:, m::G, :, :2 * d_k], g[:, ::G, :, :2 * d_k])
    np.testing.assert_array_equal(_to_oracle_state(got, H_qk, d_k, d_v), want_oracle_layout)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("with_state", [True, False])
def test_conv_frontend(dtype, with_state):
    lengths = [5, 0, 1, 2, 130, 64, 3]
    w = inputs.make_prefill(lengths, 2, 4, 32, 64, dtype=dtype, seed=5, epilogue=False)
    cw, st = inputs.make_conv_params(len(lengths), 2, 4, 32, 64, seed=5, state=with_state)
    w = to_device(w)
    cw = cw.cuda()
    st = st.cuda() if st is not None else None
    qo, ko, vo, so = gdn_conv_frontend(w.q, w.k, w.v, cw, st, cu_seqlens=w.cu_seqlens)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    rq, rk, rv, rso = _oracle_conv(w.q, w.k, w.v, cw, st, w.cu_seqlens)
    for got, ref, n in ((qo, rq, "q"), (ko, rk, "k"), (vo, rv, "v")):
        rel, mx = errors(got, ref)
        # one rounding to the input dtype (bf16: 2^-9 relative) plus fp32 arithmetic
        bound = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
        assert rel <= bound, (n, rel)
        assert mx <= bound * (np.abs(ref).max() + 1), (n, mx)
    _check_state(so, rso, 2, 32, 64)


@pytest.mark.parametrize("path,dtype,dims", [
    ("simt", torch.float32, (2, 6, 64, 32)),
    ("simt", torch.bfloat16, (2, 6, 128, 128)),
    ("tensor_split", torch.bfloat16, (2, 6, 128, 128)),
    ("tensor_single", torch.bfloat16, (2, 6, 128, 128)),
    ("auto", torch.bfloat16, (2, 6, 128, 128)),
])
def test_chunk_fwd_conv(path, dtype, dims):
    Hqk, Hv, dk, dv = dims
    lengths = [130, 1, 77] if path != "tensor_split" else [200]
    w = inputs.make_prefill(lengths, Hqk, Hv, dk, dv, dtype=dtype, seed=9, s0_std=0.1)
    cw, st = inputs.make_conv_params(len(lengths), Hqk, Hv, dk, dv, seed=9)
    w = to_device(w)
    cw, st = cw.cuda(), st.cuda()
    y, fs, so = gdn_chunk_fwd_conv(w.q, w.k, w.v, cw, w.log_alpha, w.beta, conv_state_in=st,
                                   g=w.g, norm_w=w.norm_w, initial_state=w.initial_state,
                                   cu_seqlens=w.cu_seqlens, path=path)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    rq, rk, rv, rso = _oracle_conv(w.q, w.k, w.v, cw, st, w.cu_seqlens)
    # the tensor-core path hands the front end's outputs to the scan in the
    # input dtype (bf16 activations in bf16 mode): there the oracle rounds its
    # own conv outputs to that dtype on the host before the recurrence; the
    # portable kernel takes the front end fused and keeps them in fp32
    fused = path == "simt" or (path == "auto" and not (dtype == torch.bfloat16 and dk == 128
                                                       and dv == 128))
    act = torch.float32 if fused else dtype
    rnd = lambda x: torch.tensor(x).to(act).to(torch.float32).numpy()
    y_ref, s_ref = oracle.recurrence(rnd(rq), rnd(rk), rnd(rv), w.log_alpha.cpu(), w.beta.cpu(),
                                     g=w.g.cpu().float(), norm_w=w.norm_w.cpu(),
                                     initial_state=w.initial_state.cpu(),
                                     cu_seqlens=w.cu_seqlens.cpu().long())
    assert_close(y, y_ref, dtype, "%s y" % path)
    assert_close(fs, s_ref, dtype, "%s final state" % path)
    _check_state(so, rso, Hqk, dk, dv)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T_s", [1, 2, 5])
def test_decode_conv_against_oracle(dtype, T_s):
    N, Hqk, Hv, dk, dv = 3, 2, 4, 64, 32
    d = inputs.make_decode(N=N, steps=T_s, H_qk=Hqk, H_v=Hv, d_k=dk, d_v=dv, dtype=dtype,
                           seed=T_s, epilogue=True)
    cw, cst = inputs.make_conv_params(N, Hqk, Hv, dk, dv, seed=T_s)
    tr = lambda x: x.transpose(0, 1).contiguous().cuda()  # [steps, N, ...] -> [N, T_s, ...]
    q, k, v, la, b, g = tr(d.q), tr(d.k), tr(d.v), tr(d.log_alpha), tr(d.beta), tr(d.g)
    s0 = d.state.cuda()
    state = s0.clone()
    conv_state = cst.cuda().clone()
    y, snaps = gdn_decode_conv(q, k, v, cw.cuda(), la, b, state, conv_state, snapshots=True,
                               g=g, norm_w=d.norm_w.cuda())
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    # oracle: each sequence is a packed sequence of T_s tokens
    flat = lambda x: x.reshape((N * T_s,) + tuple(x.shape[2:]))
    cu = torch.arange(0, N * T_s + 1, T_s, dtype=torch.int32)
    rq, rk, rv, rso = _oracle_conv(flat(q), flat(k), flat(v), cw, cst.cuda(), cu)
    y_ref, s_ref = oracle.recurrence(rq.astype(np.float32), rk.astype(np.float32),
                                     rv.astype(np.float32), flat(la).cpu(), flat(b).cpu(),
                                     g=flat(g).cpu().float(), norm_w=d.norm_w,
                                     initial_state=s0.cpu(), cu_seqlens=cu.long())
    tol_dtype = dtype
    assert_close(flat(y), y_ref, tol_dtype, "decode_conv y")
    assert_close(state, s_ref, torch.float32 if dtype == torch.float32 else dtype, "state")
    torch.testing.assert_close(snaps[-1], state, rtol=0, atol=0)
    _check_state(conv_state, rso, Hqk, dk, dv)


def test_decode_conv_continues_prefill_conv():
    """prefill_conv over T tokens, then decode_conv over 4 more == prefill_conv
    over all T + 4 (fp32; portable prefill kernel)."""
    Hqk, Hv, dk, dv = 2, 4, 64, 64
    T, T_s = 150, 4
    w = inputs.make_prefill([T + T_s], Hqk, Hv, dk, dv, dtype=torch.float32, seed=21,
                            s0_std=0.1)
    cw, st = inputs.make_conv_params(1, Hqk, Hv, dk, dv, seed=21)
    w = to_device(w)
    cw, st = cw.cuda(), st.cuda()
    y_all, fs_all, so_all = gdn_chunk_fwd_conv(w.q, w.k, w.v, cw, w.log_alpha, w.beta,
                                               conv_state_in=st, g=w.g, norm_w=w.norm_w,
                                               initial_state=w.initial_state, path="simt")
    y_a, fs_a, so_a = gdn_chunk_fwd_conv(w.q[:T], w.k[:T], w.v[:T], cw, w.log_alpha[:T],
                                         w.beta[:T], conv_state_in=st, g=w.g[:T],
                                         norm_w=w.norm_w, initial_state=w.initial_state,
                                         path="simt")
    u = lambda x: x[T:].unsqueeze(0).contiguous()
    state = fs_a.clone()
    conv_state = so_a.clone()
    y_b, _ = gdn_decode_conv(u(w.q), u(w.k), u(w.v), cw, u(w.log_alpha), u(w.beta), state,
                             conv_state, g=u(w.g), norm_w=w.norm_w)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    torch.testing.assert_close(conv_state, so_all, rtol=0, atol=0)
    assert_close(y_a, y_all[:T].cpu().double().numpy(), torch.float32, "prefix y")
    assert_close(y_b[0], y_all[T:].cpu().double().numpy(), torch.float32, "decoded y")
    assert_close(state, fs_all.cpu().double().numpy(), torch.float32, "state")


def test_conv_frontend_all_sequences_empty_carries_state():
    w = to_device(inputs.make_prefill([0, 0, 0], 2, 4, 16, 32, dtype=torch.float32, seed=2,
                                      epilogue=False))
    cw, st = inputs.make_conv_params(3, 2, 4, 16, 32, seed=2)
    qo, ko, vo, so = gdn_conv_frontend(w.q, w.k, w.v, cw.cuda(), st.cuda(),
                                       cu_seqlens=w.cu_seqlens)
    torch.cuda.synchronize()
    assert gdn_check_device_error() == gdn.GDN_OK
    torch.testing.assert_close(so, st.cuda(), rtol=0, atol=0)
