"""Pins for the oracle's backward (the hand-written adjoint of the error-form
recurrence, "Qwen3.8-Flash-Next: architecture, efficiency and technical
lineage", section 03 "Gated DeltaNet", update equations; epilogue from the
same section, "what Qwen changed on the original GDN").

The adjoint is checked against things that do not share its derivation:

* central finite differences of the (separately pinned) forward oracle,
  Richardson-extrapolated, for every element of every input, on tiny cases
  with and without the epilogue, the L2 norm, several sequences and a
  grouped QK head;
* reverse-mode automatic differentiation (torch.autograd, fp64) of a plain
  PyTorch restatement of the recurrence, on cases long enough to cross the
  oracle's recomputation blocks;
* closed forms for beta = 0 (pure decay): dS0, dq, dv = dk = 0 and
  dlog_alpha_t = sum_{s >= t} dy_s . y_s + dS_T . S_T.
"""
import numpy as np
import pytest
import torch

import oracle

H = 2.0 ** -8          # finite-difference step; inputs sit on a 2^-12 grid
GRID = 2.0 ** -12      # so x +- H and x +- H/2 are exact in fp32


def _q(x):
    return (np.round(np.asarray(x, np.float64) / GRID) * GRID).astype(np.float32)


def _case(T, Hqk, Hv, dk, dv, seed, lengths=None, epilogue=False, s0=True):
    r = np.random.default_rng(seed)
    lengths = lengths or [T]
    c = dict(
        q=_q(r.standard_normal((T, Hqk, dk))),
        k=_q(r.standard_normal((T, Hqk, dk))),
        v=_q(r.standard_normal((T, Hv, dv))),
        log_alpha=_q(-np.log1p(np.exp(r.standard_normal((T, Hv)))) * 0.3),
        beta=_q(0.1 + 0.8 / (1 + np.exp(-r.standard_normal((T, Hv))))),
        initial_state=_q(r.standard_normal((len(lengths), Hv, dk, dv)) * 0.3) if s0 else None,
        cu_seqlens=np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64),
    )
    if epilogue:
        c["g"] = _q(r.standard_normal((T, Hv, dv)))
        c["norm_w"] = _q(r.standard_normal(dv) * 0.2)
    cot = dict(dy=_q(r.standard_normal((T, Hv, dv))),
               d_final_state=_q(r.standard_normal((len(lengths), Hv, dk, dv))))
    return c, cot


def _loss(c, cot, **kw):
    y, fs = oracle.recurrence(**c, **kw)
    return float((y * cot["dy"]).sum() + (fs * cot["d_final_state"]).sum())


GRADS = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "dlog_alpha"),
         ("beta", "dbeta"), ("initial_state", "d_initial_state"), ("g", "dg"),
         ("norm_w", "dnorm_w")]


@pytest.mark.parametrize("kw", [
    dict(T=9, Hqk=1, Hv=2, dk=4, dv=3, epilogue=False, l2norm=True, scale=1.0),
    dict(T=9, Hqk=1, Hv=2, dk=4, dv=3, epilogue=True, l2norm=True, scale=0.7),
    dict(T=7, Hqk=2, Hv=2, dk=3, dv=4, epilogue=True, l2norm=False, scale=1.0),
    dict(T=8, Hqk=1, Hv=3, dk=3, dv=2, epilogue=False, l2norm=True, scale=1.0,
         lengths=[3, 0, 5]),
])
def test_backward_matches_finite_differences(kw):
    kw = dict(kw)
    opts = dict(l2norm=kw.pop("l2norm"), scale=kw.pop("scale"), eps_l2=1e-6, eps_norm=1e-6)
    c, cot = _case(kw.pop("T"), kw.pop("Hqk"), kw.pop("Hv"), kw.pop("dk"), kw.pop("dv"),
                   seed=7, **kw)
    got = oracle.backward(**c, **cot, **opts)
    for name, gname in GRADS:
        if c.get(name) is None:
            continue
        x = c[name]
        fd = np.zeros(x.shape)
        for idx in np.ndindex(*x.shape):
            def d(h):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                assert float(xp[idx]) - float(x[idx]) == h  # exact perturbation
                return (_loss({**c, name: xp}, cot, **opts)
                        - _loss({**c, name: xm}, cot, **opts)) / (2 * h)
            fd[idx] = (4 * d(H / 2) - d(H)) / 3
        np.testing.assert_allclose(got[gname], fd, rtol=1e-6, atol=1e-7,
                                   err_msg="gradient w.r.t. %s" % name)


def _torch_forward(c, l2norm, eps_l2, eps_norm, scale):
    """The recurrence restated in plain fp64 PyTorch (for autograd only)."""
    t = {k_: (torch.tensor(v_.astype(np.float64), requires_grad=True)
              if v_ is not None and k_ != "cu_seqlens" else v_) for k_, v_ in c.items()}
    q, k, v, la, b = t["q"], t["k"], t["v"], t["log_alpha"], t["beta"]
    Hqk, Hv = q.shape[1], v.shape[1]
    G = Hv // Hqk
    if l2norm:
        qn = q / torch.sqrt((q * q).sum(-1, keepdim=True) + eps_l2)
        kn = k / torch.sqrt((k * k).sum(-1, keepdim=True) + eps_l2)
    else:
        qn, kn = q, k
    cu = c["cu_seqlens"]
    ys, finals = [None] * q.shape[0], []
    for s in range(len(cu) - 1):
        heads = []
        for h in range(Hv):
            S = t["initial_state"][s, h]
            rows = []
            for i in range(cu[s], cu[s + 1]):
                kk, qq = kn[i, h // G], qn[i, h // G]
                S = torch.exp(la[i, h]) * S
                e = v[i, h] - S.T @ kk
                S = S + b[i, h] * torch.outer(kk, e)
                rows.append(scale * (S.T @ qq))
            heads.append((S, rows))
        finals.append(torch.stack([S for S, _ in heads]))
        for n, i in enumerate(range(cu[s], cu[s + 1])):
            ys[i] = torch.stack([rows[n] for _, rows in heads])
    y = torch.stack(ys)
    if t.get("g") is not None:
        r = 1 / torch.sqrt((y * y).mean(-1, keepdim=True) + eps_norm)
        y = y * r * (1 + t["norm_w"]) * torch.sigmoid(t["g"])
    return t, y, torch.stack(finals)


@pytest.mark.parametrize("T,lengths,epilogue", [(70, None, False), (130, [61, 69], True)])
def test_backward_matches_autograd(T, lengths, epilogue):
    c, cot = _case(T, 1, 3, 8, 6, seed=T, lengths=lengths, epilogue=epilogue)
    opts = dict(l2norm=True, eps_l2=1e-6, eps_norm=1e-6, scale=0.9)
    t, y, fs = _torch_forward(c, **opts)
    loss = (y * torch.tensor(cot["dy"], dtype=torch.float64)).sum() + \
        (fs * torch.tensor(cot["d_final_state"], dtype=torch.float64)).sum()
    loss.backward()
    got = oracle.backward(**c, **cot, **opts)
    for name, gname in GRADS:
        if c.get(name) is None:
            continue
        np.testing.assert_allclose(got[gname], t[name].grad.numpy(), rtol=1e-10, atol=1e-11,
                                   err_msg="gradient w.r.t. %s" % name)


def test_backward_beta_zero_closed_forms():
    """beta = 0: S_t = gamma_t S0 with gamma_t = exp(sum_{s<=t} log alpha_s)."""
    c, cot = _case(40, 1, 1, 5, 4, seed=3)
    c["beta"] = np.zeros_like(c["beta"])
    got = oracle.backward(**c, **cot, eps_l2=0.0)
    y, fs = oracle.recurrence(**c, eps_l2=0.0)
    S0 = c["initial_state"][0, 0].astype(np.float64)
    gam = np.exp(np.cumsum(c["log_alpha"][:, 0].astype(np.float64)))
    q = c["q"][:, 0].astype(np.float64)
    qn = q / np.linalg.norm(q, axis=1, keepdims=True)
    dy = cot["dy"][:, 0].astype(np.float64)
    dsT = cot["d_final_state"][0, 0].astype(np.float64)
    # dS0 = gamma_T dS_T + sum_t gamma_t q^_t dy_t^T
    ds0 = gam[-1] * dsT + np.einsum("t,ti,tj->ij", gam, qn, dy)
    np.testing.assert_allclose(got["d_initial_state"][0, 0], ds0, rtol=1e-12, atol=1e-12)
    assert np.abs(got["dv"]).max() == 0 and np.abs(got["dk"]).max() == 0
    # dq^_t = gamma_t S0 dy_t, then through the L2 norm
    dqn = gam[:, None] * (dy @ S0.T)
    r = 1 / np.linalg.norm(q, axis=1, keepdims=True)
    dq = r * (dqn - qn * (qn * dqn).sum(1, keepdims=True))
    np.testing.assert_allclose(got["dq"][:, 0], dq, rtol=1e-11, atol=1e-12)
    # every y_s and S_T scale with gamma, so dlog alpha_t = sum_{s>=t} dy_s.y_s + dS_T.S_T
    contrib = (dy * y[:, 0]).sum(1)
    dla = np.cumsum(contrib[::-1])[::-1] + (dsT * fs[0, 0]).sum()
    np.testing.assert_allclose(got["dlog_alpha"][:, 0], dla, rtol=1e-11, atol=1e-12)
