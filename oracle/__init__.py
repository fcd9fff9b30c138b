"""fp64 CPU oracle for the gated delta rule (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it shares no code
with that path.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, OpenMP over
(sequence, value head) pairs); this module only compiles it with gcc and
marshals numpy arrays.  What it computes, and which page each step follows, is
stated at the top of ``gdn_oracle.c``:

* the error form of the gated delta rule, token by token
  ("Qwen3.8-Flash-Next: architecture, efficiency and technical lineage",
  section 03 "Gated DeltaNet", update equations);
* the product form alpha (I - beta k k^T) S + beta k v^T
  ("On the Design of Qwen3.8-Next Architecture ... close reading",
  section 4.1), used only to pin the error form;
* the optional zero-centred RMSNorm x sigmoid(g) epilogue (section 03,
  "what Qwen changed on the original GDN"; hyper.ai summary, "Method");
* the front end: short depthwise causal convolution (kernel 4) and SiLU
  (section 02 module table, GDN row; hyper.ai "Method"; close reading 4.1);
* the backward of all of the above (the adjoint of the error-form recurrence,
  differentiated by hand token by token in reverse order), for training.

The pins that tie each function to the pages and to mathematics other than
itself are in ``tests/test_oracle_pins.py`` (the recurrence, both forms, the
epilogue), ``tests/test_oracle_conv_pins.py`` (the front end) and
``tests/test_oracle_backward_pins.py`` (the backward); the Gated Residual
oracle (``oracle/gr.py``) is pinned in ``tests/test_oracle_gr_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.gdn_oracle_recurrence.restype = ctypes.c_int
        lib.gdn_oracle_recurrence.argtypes = [
            _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _i64p,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_double, ctypes.c_double, _f64p, _f64p, ctypes.c_int]
        lib.gdn_oracle_product_form.restype = ctypes.c_int
        lib.gdn_oracle_product_form.argtypes = [
            _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int64,
            ctypes.c_int, ctypes.c_int, _f64p, _f64p]
        lib.gdn_oracle_backward.restype = ctypes.c_int
        lib.gdn_oracle_backward.argtypes = [
            _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _i64p,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_double, ctypes.c_double, _f32p, _f32p, _f64p, _f64p,
            _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int]
        lib.gdn_oracle_conv.restype = ctypes.c_int
        lib.gdn_oracle_conv.argtypes = [
            _f32p, ctypes.c_int64, ctypes.c_int, _f32p, _f32p, _i64p, ctypes.c_int64,
            ctypes.c_int, _f64p, _f64p]
        lib.gdn_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _as_np(x, dtype):
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor: widen on the CPU, exactly
        import torch
        x = x.detach().to("cpu", torch.float64 if dtype == np.float64 else torch.float32)
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def _ptr(a, typ):
    return None if a is None else a.ctypes.data_as(typ)


def max_threads() -> int:
    return int(_load().gdn_oracle_max_threads())


def recurrence(q, k, v, log_alpha, beta, g=None, norm_w=None,
               initial_state=None, cu_seqlens=None, l2norm=True,
               eps_l2=1e-6, eps_norm=1e-6, scale=1.0, n_threads=0):
    """Error-form gated delta rule over a packed batch, in fp64.

    Shapes: q, k [T, H_qk, d_k]; v [T, H_v, d_v]; log_alpha, beta [T, H_v];
    g [T, H_v, d_v] or None; norm_w [d_v] or None; initial_state
    [n_seq, H_v, d_k, d_v] or None (zeros); cu_seqlens [n_seq + 1] or None
    (one sequence).  Inputs are widened exactly to fp32 then fp64.
    Returns (y [T, H_v, d_v], final_state [n_seq, H_v, d_k, d_v]) as float64.
    """
    lib = _load()
    q = _as_np(q, np.float32)
    k = _as_np(k, np.float32)
    v = _as_np(v, np.float32)
    la = _as_np(log_alpha, np.float32)
    b = _as_np(beta, np.float32)
    g = _as_np(g, np.float32)
    w = _as_np(norm_w, np.float32)
    s0 = _as_np(initial_state, np.float32)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = _as_np(cu_seqlens, np.int64)
    n_seq = cu.shape[0] - 1
    y = np.zeros((T, Hv, dv), dtype=np.float64)
    fs = np.zeros((n_seq, Hv, dk, dv), dtype=np.float64)
    rc = lib.gdn_oracle_recurrence(
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(la, _f32p),
        _ptr(b, _f32p), _ptr(g, _f32p), _ptr(w, _f32p), _ptr(s0, _f32p),
        _ptr(cu, _i64p), n_seq, T, Hqk, Hv, dk, dv, int(bool(l2norm)),
        float(eps_l2), float(eps_norm), float(scale), _ptr(y, _f64p),
        _ptr(fs, _f64p), int(n_threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, fs


def product_form(q, k, v, alpha, beta, s0=None):
    """Product form S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T.

    One sequence, one head, fp64 inputs used as given (no L2 norm):
    q, k [T, d_k]; v [T, d_v]; alpha, beta [T]; s0 [d_k, d_v] or None.
    Returns (y [T, d_v] with y_t = S_t^T q_t, S_T [d_k, d_v]).
    """
    lib = _load()
    q = _as_np(q, np.float64)
    k = _as_np(k, np.float64)
    v = _as_np(v, np.float64)
    a = _as_np(alpha, np.float64)
    b = _as_np(beta, np.float64)
    s0 = _as_np(s0, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    y = np.zeros((T, dv), dtype=np.float64)
    s = np.zeros((dk, dv), dtype=np.float64)
    rc = lib.gdn_oracle_product_form(
        _ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p), _ptr(a, _f64p),
        _ptr(b, _f64p), _ptr(s0, _f64p), T, dk, dv, _ptr(y, _f64p),
        _ptr(s, _f64p))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, s


def backward(q, k, v, log_alpha, beta, dy, g=None, norm_w=None,
             initial_state=None, d_final_state=None, cu_seqlens=None,
             l2norm=True, eps_l2=1e-6, eps_norm=1e-6, scale=1.0, n_threads=0):
    """Gradients of sum(dy * y) + sum(d_final_state * final_state) with
    respect to every input of ``recurrence``, in fp64.

    dy has the shape of y ([T, H_v, d_v]; the gradient after the epilogue when
    g is given); d_final_state [n_seq, H_v, d_k, d_v] or None (zeros).  Inputs
    are widened exactly to fp32 then fp64.  Returns a dict with dq, dk
    [T, H_qk, d_k]; dv [T, H_v, d_v]; dlog_alpha, dbeta [T, H_v];
    d_initial_state [n_seq, H_v, d_k, d_v]; and, when g is given, dg
    [T, H_v, d_v] and dnorm_w [d_v].
    """
    lib = _load()
    q = _as_np(q, np.float32)
    k = _as_np(k, np.float32)
    v = _as_np(v, np.float32)
    la = _as_np(log_alpha, np.float32)
    b = _as_np(beta, np.float32)
    g = _as_np(g, np.float32)
    w = _as_np(norm_w, np.float32)
    s0 = _as_np(initial_state, np.float32)
    dyy = _as_np(dy, np.float32)
    dsT = _as_np(d_final_state, np.float32)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    cu = (np.array([0, T], dtype=np.int64) if cu_seqlens is None
          else _as_np(cu_seqlens, np.int64))
    n_seq = cu.shape[0] - 1
    out = dict(dq=np.zeros((T, Hqk, dk)), dk=np.zeros((T, Hqk, dk)),
               dv=np.zeros((T, Hv, dv)), dlog_alpha=np.zeros((T, Hv)),
               dbeta=np.zeros((T, Hv)), d_initial_state=np.zeros((n_seq, Hv, dk, dv)))
    if g is not None:
        out["dg"] = np.zeros((T, Hv, dv))
        out["dnorm_w"] = np.zeros(dv)
    rc = lib.gdn_oracle_backward(
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(la, _f32p),
        _ptr(b, _f32p), _ptr(g, _f32p), _ptr(w, _f32p), _ptr(s0, _f32p),
        _ptr(cu, _i64p), n_seq, T, Hqk, Hv, dk, dv, int(bool(l2norm)),
        float(eps_l2), float(eps_norm), float(scale), _ptr(dyy, _f32p),
        _ptr(dsT, _f32p), _ptr(out["dq"], _f64p), _ptr(out["dk"], _f64p),
        _ptr(out["dv"], _f64p), _ptr(out["dlog_alpha"], _f64p),
        _ptr(out["dbeta"], _f64p), _ptr(out.get("dg"), _f64p),
        _ptr(out.get("dnorm_w"), _f64p), _ptr(out["d_initial_state"], _f64p),
        int(n_threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def conv(x, w, state_in=None, cu_seqlens=None, silu=True):
    """Depthwise causal convolution of kernel 4 over time, then SiLU, in fp64.

    x [T, C]; w [C, 4] (w[:, 3] weighs the current token); state_in
    [n_seq, 3, C] or None (zeros): the three inputs before each sequence's
    first token, oldest first.  Returns (y [T, C], state_out [n_seq, 3, C]),
    state_out holding the last three inputs of each sequence, oldest first.
    """
    lib = _load()
    xx = _as_np(x, np.float32)
    ww = _as_np(w, np.float32)
    st = _as_np(state_in, np.float32)
    T, C = xx.shape
    cu = (np.array([0, T], dtype=np.int64) if cu_seqlens is None
          else _as_np(cu_seqlens, np.int64))
    n_seq = cu.shape[0] - 1
    y = np.zeros((T, C), dtype=np.float64)
    so = np.zeros((n_seq, 3, C), dtype=np.float64)
    rc = lib.gdn_oracle_conv(_ptr(xx, _f32p), T, C, _ptr(ww, _f32p), _ptr(st, _f32p),
                             _ptr(cu, _i64p), n_seq, int(bool(silu)), _ptr(y, _f64p),
                             _ptr(so, _f64p))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, so
