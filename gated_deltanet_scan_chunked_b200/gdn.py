"""Thin Python binding of libgdn (see include/gdn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libgdn.so.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or the tensors are
not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "gdn.h")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = range(5)
GDN_BF16, GDN_FP32 = 0, 1
PATHS = {"auto": 0, "tensor": 1, "simt": 2, "tensor_pair": 3, "tensor_single": 4,
         "tensor_split": 5}
# paths that may run the split layout, which needs a workspace
_WS_PATHS = ("auto", "tensor", "tensor_split")

_lib = None
_vp = ctypes.c_void_p


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


def load(path: str = LIB_PATH):
    """Load libgdn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            "libgdn.so not found at %s; build it with "
            "`python -m gated_deltanet_scan_chunked_b200.build`" % path)
    lib = ctypes.CDLL(path)
    f = lib.gdn_chunk_fwd_path
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 9 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp,
        ctypes.c_int, _vp]
    f = lib.gdn_chunk_fwd_ws
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 9 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp,
        ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    f = lib.gdn_chunk_fwd_static_ws
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 9 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp, _vp]
    f = lib.gdn_chunk_fwd_workspace_size
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int32] * 4 + [ctypes.c_int]
    f = lib.gdn_chunk_fwd
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 9 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp, _vp]
    f = lib.gdn_decode_step
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 8 + [ctypes.c_int32] * 6 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp]
    f = lib.gdn_decode_multi
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 10 + [ctypes.c_int32] * 7 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp]
    f = lib.gdn_chunk_bwd_workspace_size
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 4
    f = lib.gdn_chunk_bwd
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 9 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float] + [_vp] * 10 + [
        _vp, ctypes.c_size_t, _vp]
    f = lib.gdn_conv_frontend
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 7 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        _vp, _vp, _vp, _vp]
    f = lib.gdn_chunk_fwd_conv_workspace_size
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 4 + [ctypes.c_int]
    f = lib.gdn_chunk_fwd_conv
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 12 + [ctypes.c_int32, ctypes.c_int64] + [ctypes.c_int32] * 5 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp,
        ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    f = lib.gdn_decode_conv
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 12 + [ctypes.c_int32] * 7 + [
        ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp]
    f = lib.gdn_gr_read_workspace_size
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    f = lib.gdn_gr_read
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 6 + [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                              ctypes.c_float, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    f = lib.gdn_gr_write
    f.restype = ctypes.c_int
    f.argtypes = [_vp] * 4 + [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _vp]
    lib.gdn_selftest_bounded_wait.restype = ctypes.c_int
    lib.gdn_selftest_bounded_wait.argtypes = [ctypes.c_int32, _vp]
    lib.gdn_check_device_error.restype = ctypes.c_int
    lib.gdn_check_device_error.argtypes = [_vp]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_status_string.argtypes = [ctypes.c_int]
    lib.gdn_version.restype = ctypes.c_int32
    lib.gdn_version.argtypes = []
    _lib = lib
    return lib


def header_functions(path: str = HEADER_PATH):
    """Names of the functions declared in include/gdn.h."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code_of(dtype) -> int:
    if dtype == torch.bfloat16:
        return GDN_BF16
    if dtype == torch.float32:
        return GDN_FP32
    raise TypeError("q/k/v/g must be bfloat16 or float32, got %s" % dtype)


def _dtype_code(t: torch.Tensor) -> int:
    return _dtype_code_of(t.dtype)


def _check(t: Optional[torch.Tensor], name: str, dtype=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (libgdn has no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))


def workspace_size(n_seq: int, H_v: int, d_k: int, d_v: int, dtype=torch.bfloat16) -> int:
    """Bytes of workspace the split prefill layout uses (0: not applicable)."""
    return int(load().gdn_chunk_fwd_workspace_size(n_seq, H_v, d_k, d_v, _dtype_code_of(dtype)))


def gdn_chunk_fwd(q, k, v, log_alpha, beta, g=None, norm_w=None,
                  initial_state=None, cu_seqlens=None, l2norm_qk=True,
                  eps_l2=1e-6, eps_norm=1e-6, scale=1.0, y=None,
                  final_state=None, output_final_state=True, path="auto",
                  workspace="auto", stream=None
                  ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked prefill over packed sequences: returns (y, final_state).

    q, k [T, H_qk, d_k]; v [T, H_v, d_v]; log_alpha, beta [T, H_v] fp32;
    g [T, H_v, d_v] or None; norm_w [d_v] fp32 or None; initial_state
    [n_seq, H_v, d_k, d_v] fp32 or None; cu_seqlens [n_seq + 1] int32 (device)
    or None.  y / final_state may be passed in (final_state may be
    initial_state itself for an in-place update).  ``workspace``: a uint8
    CUDA tensor of at least ``workspace_size(...)`` bytes, None (no split
    layout), or "auto" (allocated here through torch when the path may use
    it).  A workspace must not be shared by calls that can overlap.
    """
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    n_seq = 1 if cu_seqlens is None else int(cu_seqlens.shape[0]) - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g)):
        _check(t, name, q.dtype, dev)
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("norm_w", norm_w),
                    ("initial_state", initial_state)):
        _check(t, name, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if y is None:
        y = torch.empty((T, Hv, dv), dtype=q.dtype, device=dev)
    _check(y, "y", q.dtype, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((n_seq, Hv, dk, dv), dtype=torch.float32, device=dev)
    _check(final_state, "final_state", torch.float32, dev)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be a tensor, None or 'auto'")
        workspace = None
        if path in _WS_PATHS:
            nbytes = int(lib.gdn_chunk_fwd_workspace_size(n_seq, Hv, dk, dv, dt))
            if nbytes > 0:
                workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8, dev)
    ws_bytes = 0 if workspace is None else workspace.numel()
    st = lib.gdn_chunk_fwd_ws(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(g), _ptr(norm_w),
        _ptr(initial_state), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, dk, dv, dt,
        1 if l2norm_qk else 0, float(eps_l2), float(eps_norm), float(scale), _ptr(y),
        _ptr(final_state), PATHS[path], _ptr(workspace), ws_bytes, _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd")
    return y, final_state


def gdn_chunk_fwd_static_ws(q, k, v, log_alpha, beta, g=None, norm_w=None,
                            initial_state=None, cu_seqlens=None, l2norm_qk=True,
                            eps_l2=1e-6, eps_norm=1e-6, scale=1.0, y=None,
                            final_state=None, output_final_state=True, stream=None
                            ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The split-layout prefill with the library's own fixed workspace (at
    most 48 sequence x head items); arguments and results as gdn_chunk_fwd.
    Calls that can overlap must not be made (they share that workspace)."""
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    n_seq = 1 if cu_seqlens is None else int(cu_seqlens.shape[0]) - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g)):
        _check(t, name, q.dtype, dev)
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("norm_w", norm_w),
                    ("initial_state", initial_state)):
        _check(t, name, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if y is None:
        y = torch.empty((T, Hv, dv), dtype=q.dtype, device=dev)
    _check(y, "y", q.dtype, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((n_seq, Hv, dk, dv), dtype=torch.float32, device=dev)
    _check(final_state, "final_state", torch.float32, dev)
    st = lib.gdn_chunk_fwd_static_ws(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(g), _ptr(norm_w),
        _ptr(initial_state), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, dk, dv, dt,
        1 if l2norm_qk else 0, float(eps_l2), float(eps_norm), float(scale), _ptr(y),
        _ptr(final_state), _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_static_ws")
    return y, final_state


def bwd_workspace_size(n_seq: int, total_T: int, H_qk: int, H_v: int, d_k: int,
                       d_v: int) -> int:
    """Bytes of workspace gdn_chunk_bwd needs (0: arguments it never accepts)."""
    return int(load().gdn_chunk_bwd_workspace_size(n_seq, total_T, H_qk, H_v, d_k, d_v))


def gdn_chunk_bwd(q, k, v, log_alpha, beta, dy, g=None, norm_w=None,
                  initial_state=None, d_final_state=None, cu_seqlens=None,
                  l2norm_qk=True, eps_l2=1e-6, eps_norm=1e-6, scale=1.0,
                  want_d_initial_state=True, want_dnorm_w=True, workspace=None,
                  stream=None) -> dict:
    """Gradients of a gdn_chunk_fwd call with the same inputs.

    dy [T, H_v, d_v] (dtype of q): gradient with respect to y; d_final_state
    [n_seq, H_v, d_k, d_v] fp32 or None.  Returns a dict of fp32 tensors: dq,
    dk [T, H_qk, d_k]; dv [T, H_v, d_v]; dlog_alpha, dbeta [T, H_v]; and
    d_initial_state [n_seq, H_v, d_k, d_v], dg [T, H_v, d_v], dnorm_w [d_v]
    when asked for / when g is given.  ``workspace``: a uint8 CUDA tensor of
    at least ``bwd_workspace_size(...)`` bytes, or None (allocated here
    through torch).
    """
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    n_seq = 1 if cu_seqlens is None else int(cu_seqlens.shape[0]) - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("dy", dy)):
        _check(t, name, q.dtype, dev)
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("norm_w", norm_w),
                    ("initial_state", initial_state), ("d_final_state", d_final_state)):
        _check(t, name, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty((T, Hqk, dk), **f32), dk=torch.empty((T, Hqk, dk), **f32),
               dv=torch.empty((T, Hv, dv), **f32), dlog_alpha=torch.empty((T, Hv), **f32),
               dbeta=torch.empty((T, Hv), **f32))
    if want_d_initial_state:
        out["d_initial_state"] = torch.empty((n_seq, Hv, dk, dv), **f32)
    if g is not None:
        out["dg"] = torch.empty((T, Hv, dv), **f32)
        if want_dnorm_w:
            out["dnorm_w"] = torch.empty((dv,), **f32)
    nbytes = int(lib.gdn_chunk_bwd_workspace_size(n_seq, T, Hqk, Hv, dk, dv))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8, dev)
    st = lib.gdn_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(g), _ptr(norm_w),
        _ptr(initial_state), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, dk, dv, dt,
        1 if l2norm_qk else 0, float(eps_l2), float(eps_norm), float(scale), _ptr(dy),
        _ptr(d_final_state), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
        _ptr(out["dlog_alpha"]), _ptr(out["dbeta"]), _ptr(out.get("dg")),
        _ptr(out.get("dnorm_w")), _ptr(out.get("d_initial_state")), _ptr(workspace),
        workspace.numel(), _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_bwd")
    return out


def gdn_decode_step(q, k, v, log_alpha, beta, state, g=None, norm_w=None,
                    l2norm_qk=True, eps_l2=1e-6, eps_norm=1e-6, scale=1.0,
                    y=None, stream=None) -> torch.Tensor:
    """One token per sequence; ``state`` [N, H_v, d_k, d_v] fp32 is updated
    in place.  q, k [N, H_qk, d_k]; v [N, H_v, d_v]; gates [N, H_v].
    Returns y [N, H_v, d_v]."""
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    N, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g)):
        _check(t, name, q.dtype, dev)
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("norm_w", norm_w),
                    ("state", state)):
        _check(t, name, torch.float32, dev)
    if y is None:
        y = torch.empty((N, Hv, dv), dtype=q.dtype, device=dev)
    _check(y, "y", q.dtype, dev)
    st = lib.gdn_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(g), _ptr(norm_w),
        _ptr(state), N, Hqk, Hv, dk, dv, dt, 1 if l2norm_qk else 0, float(eps_l2),
        float(eps_norm), float(scale), _ptr(y), _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_step")
    return y


def gdn_decode_multi(q, k, v, log_alpha, beta, state_in, state_out="in_place",
                     snapshots=None, g=None, norm_w=None, l2norm_qk=True, eps_l2=1e-6,
                     eps_norm=1e-6, scale=1.0, y=None, stream=None) -> torch.Tensor:
    """T_s tokens per sequence in one launch.  q, k [N, T_s, H_qk, d_k];
    v [N, T_s, H_v, d_v]; gates [N, T_s, H_v]; state_in [N, H_v, d_k, d_v]
    fp32.  state_out: "in_place" (default: state_in is updated), a tensor, or
    None (not written).  snapshots: None, True (allocated here), or a
    [T_s, N, H_v, d_k, d_v] fp32 tensor receiving the state after each
    token.  Returns (y, snapshots)."""
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    N, T_s, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g)):
        _check(t, name, q.dtype, dev)
    if isinstance(state_out, str):
        if state_out != "in_place":
            raise ValueError("state_out must be a tensor, None or 'in_place'")
        state_out = state_in
    if snapshots is True:
        snapshots = torch.empty((T_s, N, Hv, dk, dv), dtype=torch.float32, device=dev)
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("norm_w", norm_w),
                    ("state_in", state_in), ("state_out", state_out),
                    ("snapshots", snapshots)):
        _check(t, name, torch.float32, dev)
    if y is None:
        y = torch.empty((N, T_s, Hv, dv), dtype=q.dtype, device=dev)
    _check(y, "y", q.dtype, dev)
    st = lib.gdn_decode_multi(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(g), _ptr(norm_w),
        _ptr(state_in), _ptr(state_out), _ptr(snapshots), N, T_s, Hqk, Hv, dk, dv, dt,
        1 if l2norm_qk else 0, float(eps_l2), float(eps_norm), float(scale), _ptr(y),
        _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_multi")
    return y, snapshots


def conv_state_shape(n_seq: int, H_v: int, d_k: int, d_v: int):
    """Shape of the carried conv state: [n_seq, H_v, 3, 2 d_k + d_v]."""
    return (n_seq, H_v, 3, 2 * d_k + d_v)


def gdn_conv_frontend(q, k, v, conv_w, conv_state_in=None, cu_seqlens=None,
                      conv_state_out=True, out=None, stream=None):
    """Causal depthwise conv (kernel 4) + SiLU over q, k, v (pre-conv, shapes
    as gdn_chunk_fwd).  conv_w [2 H_qk d_k + H_v d_v, 4] fp32 (channels q |
    k | v); conv_state_in [n_seq, H_v, 3, 2 d_k + d_v] fp32 or None;
    conv_state_out: True (allocated here), a tensor, or None (not written).
    Returns (q', k', v', conv_state_out)."""
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    n_seq = 1 if cu_seqlens is None else int(cu_seqlens.shape[0]) - 1
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, q.dtype, dev)
    if conv_state_out is True:
        conv_state_out = torch.empty(conv_state_shape(n_seq, Hv, dk, dv), dtype=torch.float32,
                                     device=dev)
    for name, t in (("conv_w", conv_w), ("conv_state_in", conv_state_in),
                    ("conv_state_out", conv_state_out)):
        _check(t, name, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    qo, ko, vo = out if out is not None else (torch.empty_like(q), torch.empty_like(k),
                                              torch.empty_like(v))
    st = lib.gdn_conv_frontend(
        _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), _ptr(conv_state_in), _ptr(conv_state_out),
        _ptr(cu_seqlens), n_seq, T, Hqk, Hv, dk, dv, dt, _ptr(qo), _ptr(ko), _ptr(vo),
        _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_conv_frontend")
    return qo, ko, vo, conv_state_out


def conv_workspace_size(n_seq: int, total_T: int, H_qk: int, H_v: int, d_k: int, d_v: int,
                        dtype=torch.bfloat16) -> int:
    """Bytes of workspace gdn_chunk_fwd_conv needs (0: never accepted)."""
    return int(load().gdn_chunk_fwd_conv_workspace_size(n_seq, total_T, H_qk, H_v, d_k, d_v,
                                                        _dtype_code_of(dtype)))


def gdn_chunk_fwd_conv(q, k, v, conv_w, log_alpha, beta, conv_state_in=None,
                       conv_state_out=True, g=None, norm_w=None, initial_state=None,
                       cu_seqlens=None, l2norm_qk=True, eps_l2=1e-6, eps_norm=1e-6,
                       scale=1.0, y=None, final_state=None, output_final_state=True,
                       path="auto", workspace=None, stream=None):
    """Prefill on pre-conv q, k, v: the front end, then gdn_chunk_fwd.
    Returns (y, final_state, conv_state_out).  ``workspace``: a uint8 CUDA
    tensor of at least conv_workspace_size(...) bytes, or None (allocated)."""
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    n_seq = 1 if cu_seqlens is None else int(cu_seqlens.shape[0]) - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g)):
        _check(t, name, q.dtype, dev)
    if conv_state_out is True:
        conv_state_out = torch.empty(conv_state_shape(n_seq, Hv, dk, dv), dtype=torch.float32,
                                     device=dev)
    for name, t in (("conv_w", conv_w), ("conv_state_in", conv_state_in),
                    ("conv_state_out", conv_state_out), ("log_alpha", log_alpha),
                    ("beta", beta), ("norm_w", norm_w), ("initial_state", initial_state)):
        _check(t, name, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if y is None:
        y = torch.empty((T, Hv, dv), dtype=q.dtype, device=dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((n_seq, Hv, dk, dv), dtype=torch.float32, device=dev)
    _check(y, "y", q.dtype, dev)
    _check(final_state, "final_state", torch.float32, dev)
    nbytes = int(lib.gdn_chunk_fwd_conv_workspace_size(n_seq, T, Hqk, Hv, dk, dv, dt))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8, dev)
    st = lib.gdn_chunk_fwd_conv(
        _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), _ptr(conv_state_in), _ptr(conv_state_out),
        _ptr(log_alpha), _ptr(beta), _ptr(g), _ptr(norm_w), _ptr(initial_state),
        _ptr(cu_seqlens), n_seq, T, Hqk, Hv, dk, dv, dt, 1 if l2norm_qk else 0,
        float(eps_l2), float(eps_norm), float(scale), _ptr(y), _ptr(final_state), PATHS[path],
        _ptr(workspace), workspace.numel(), _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_conv")
    return y, final_state, conv_state_out


def gdn_decode_conv(q, k, v, conv_w, log_alpha, beta, state_in, conv_state,
                    state_out="in_place", snapshots=None, g=None, norm_w=None,
                    l2norm_qk=True, eps_l2=1e-6, eps_norm=1e-6, scale=1.0, y=None,
                    stream=None):
    """gdn_decode_multi on pre-conv q, k, v with the front end fused: q, k
    [N, T_s, H_qk, d_k]; v [N, T_s, H_v, d_v]; conv_state [N, H_v, 3,
    2 d_k + d_v] fp32, updated in place (None: zeros, not written).  Returns
    (y, snapshots)."""
    lib = load()
    dev = q.device
    dt = _dtype_code(q)
    N, T_s, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g)):
        _check(t, name, q.dtype, dev)
    if isinstance(state_out, str):
        if state_out != "in_place":
            raise ValueError("state_out must be a tensor, None or 'in_place'")
        state_out = state_in
    if snapshots is True:
        snapshots = torch.empty((T_s, N, Hv, dk, dv), dtype=torch.float32, device=dev)
    for name, t in (("conv_w", conv_w), ("conv_state", conv_state), ("log_alpha", log_alpha),
                    ("beta", beta), ("norm_w", norm_w), ("state_in", state_in),
                    ("state_out", state_out), ("snapshots", snapshots)):
        _check(t, name, torch.float32, dev)
    if y is None:
        y = torch.empty((N, T_s, Hv, dv), dtype=q.dtype, device=dev)
    _check(y, "y", q.dtype, dev)
    st = lib.gdn_decode_conv(
        _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), _ptr(conv_state), _ptr(log_alpha),
        _ptr(beta), _ptr(g), _ptr(norm_w), _ptr(state_in), _ptr(state_out), _ptr(snapshots),
        N, T_s, Hqk, Hv, dk, dv, dt, 1 if l2norm_qk else 0, float(eps_l2), float(eps_norm),
        float(scale), _ptr(y), _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_conv")
    return y, snapshots


def gr_read_workspace_size(T: int, n_r: int, d: int, rank: int) -> int:
    return int(load().gdn_gr_read_workspace_size(T, n_r, d, rank))


def gdn_gr_read(codes, scales, gamma, W_d, W_u, W_w, eps=1e-6, x=None, s=None,
                workspace=None, stream=None):
    """Gated Residual read: codes [T, n_r, d] uint8 (E4M3), scales [T, n_r]
    fp32, gamma [n_r, d] fp32, W_d [rank, n_r d], W_u [n_r d, rank], W_w
    [n_r, n_r d] bf16.  Returns (x [T, d] bf16, s [T, n_r] fp32)."""
    lib = load()
    dev = codes.device
    T, n_r, d = codes.shape
    rank = W_d.shape[0]
    _check(codes, "codes", torch.uint8, dev)
    for name, t in (("scales", scales), ("gamma", gamma)):
        _check(t, name, torch.float32, dev)
    for name, t in (("W_d", W_d), ("W_u", W_u), ("W_w", W_w)):
        _check(t, name, torch.bfloat16, dev)
    if x is None:
        x = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    if s is None:
        s = torch.empty((T, n_r), dtype=torch.float32, device=dev)
    nbytes = int(lib.gdn_gr_read_workspace_size(T, n_r, d, rank))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    st = lib.gdn_gr_read(_ptr(codes), _ptr(scales), _ptr(gamma), _ptr(W_d), _ptr(W_u),
                         _ptr(W_w), T, n_r, d, rank, float(eps), _ptr(x), _ptr(s),
                         _ptr(workspace), workspace.numel(), _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_gr_read")
    return x, s


def gdn_gr_write(codes, scales, y, s, stream=None):
    """Gated Residual write, in place: R'_i = R_i + s_i y, requantised."""
    lib = load()
    dev = codes.device
    T, n_r, d = codes.shape
    _check(codes, "codes", torch.uint8, dev)
    _check(scales, "scales", torch.float32, dev)
    _check(y, "y", torch.bfloat16, dev)
    _check(s, "s", torch.float32, dev)
    st = lib.gdn_gr_write(_ptr(codes), _ptr(scales), _ptr(y), _ptr(s), T, n_r, d,
                          _stream_handle(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_gr_write")
    return codes, scales


def gdn_check_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(load().gdn_check_device_error(_stream_handle(stream)))
