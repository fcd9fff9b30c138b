"""Pins for the oracle's front end (short depthwise causal convolution of
kernel 4, then SiLU): "Qwen3.8-Flash-Next: architecture, efficiency and
technical lineage", section 02 module table, GDN row; hyper.ai summary,
"Method"; "On the Design of Qwen3.8-Next Architecture ... close reading",
section 4.1.

Checked against library routines and exact special cases:
* torch.nn.functional.conv1d (groups = channels, left padding = the carried
  state) for the convolution, torch.nn.functional.silu for the activation;
* identity and pure-shift kernels;
* splitting a sequence and carrying the conv state == one pass (bitwise);
* packed sequences == each alone, including sequences shorter than the
  kernel (the carried state then mixes the old state and the new inputs).
"""
import numpy as np
import pytest
import torch

import oracle


def _case(T, C, seed, n_seq=1):
    r = np.random.default_rng(seed)
    x = r.standard_normal((T, C)).astype(np.float32)
    w = (r.standard_normal((C, 4)) * 0.5).astype(np.float32)
    st = r.standard_normal((n_seq, 3, C)).astype(np.float32)
    return x, w, st


def _torch_conv(x, w, st):
    xt = torch.tensor(np.concatenate([st, x], 0).T[None].astype(np.float64))  # [1, C, 3 + T]
    wt = torch.tensor(w.astype(np.float64))[:, None, :]                       # [C, 1, 4]
    return torch.nn.functional.conv1d(xt, wt, groups=x.shape[1])[0].T.numpy()  # [T, C]


@pytest.mark.parametrize("T,C", [(1, 3), (5, 7), (40, 16)])
def test_conv_matches_conv1d_and_silu(T, C):
    x, w, st = _case(T, C, T + C)
    u, so = oracle.conv(x, w, st, silu=False)
    np.testing.assert_allclose(u, _torch_conv(x, w, st[0]), rtol=1e-13, atol=1e-13)
    y, _ = oracle.conv(x, w, st, silu=True)
    np.testing.assert_allclose(y, torch.nn.functional.silu(torch.tensor(u)).numpy(),
                               rtol=1e-13, atol=1e-14)
    # zero state == zero padding
    u0, _ = oracle.conv(x, w, None, silu=False)
    np.testing.assert_allclose(u0, _torch_conv(x, w, np.zeros_like(st[0])), rtol=1e-13,
                               atol=1e-13)
    # carried state = last three inputs (oldest first), from the old state if T < 3
    np.testing.assert_array_equal(so[0], np.concatenate([st[0], x], 0)[-3:])


def test_identity_and_shift_kernels():
    x, _, st = _case(9, 4, 1)
    ident = np.zeros((4, 4), np.float32)
    ident[:, 3] = 1
    u, _ = oracle.conv(x, ident, st, silu=False)
    np.testing.assert_array_equal(u, x)
    shift = np.zeros((4, 4), np.float32)
    shift[:, 0] = 1  # the input three tokens back
    u, _ = oracle.conv(x, shift, st, silu=False)
    np.testing.assert_array_equal(u[3:], x[:-3])
    np.testing.assert_array_equal(u[:3], st[0])


@pytest.mark.parametrize("cut", [1, 2, 3, 17])
def test_split_and_carry_equals_one_pass(cut):
    x, w, st = _case(30, 6, cut)
    y, so = oracle.conv(x, w, st)
    ya, sa = oracle.conv(x[:cut], w, st)
    yb, sb = oracle.conv(x[cut:], w, sa.astype(np.float32))
    np.testing.assert_array_equal(np.concatenate([ya, yb]), y)
    np.testing.assert_array_equal(sb, so)


def test_packed_sequences_are_independent():
    lengths = [4, 0, 1, 2, 9]
    T, C = sum(lengths), 5
    x, w, st = _case(T, C, 3, n_seq=len(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    y, so = oracle.conv(x, w, st, cu_seqlens=cu)
    for s, L in enumerate(lengths):
        ys, ss = oracle.conv(x[cu[s]:cu[s + 1]], w, st[s:s + 1])
        np.testing.assert_array_equal(y[cu[s]:cu[s + 1]], ys)
        np.testing.assert_array_equal(so[s], ss[0])
