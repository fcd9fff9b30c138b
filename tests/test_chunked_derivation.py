"""The chunkwise-parallel form used by the CUDA prefill kernels, checked in
fp64 against the token-by-token oracle.

The pages give only the recurrence (error form, section 03 "Gated DeltaNet" of
"Qwen3.8-Flash-Next: architecture, efficiency and technical lineage").  The
chunked form below is derived from it: within a chunk with entering state S0,
G_t = sum_{s<=t} log alpha_s, gamma_t = exp(G_t),

  A_ti  = beta_t exp(G_t - G_i) (k_t . k_i)   for i < t, else 0
  T     = (I + A)^{-1}                        (unit lower triangular)
  W     = T diag(beta gamma) K                U = T diag(beta) V
  Delta = U - W S0                            (the values each token writes)
  Y     = diag(gamma) Q S0 + (Q K^T o M) Delta,  M_ti = exp(G_t - G_i), i <= t
  S     = gamma_C S0 + (diag(exp(G_C - G)) K)^T Delta

This test keeps that algebra honest before any kernel relies on it.
"""
import numpy as np
import pytest

import oracle


def _chunked(qh, kh, v, la, b, S0, C):
    T, dk = kh.shape
    S = S0.copy()
    ys = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        K, Q, V = kh[c0:c1], qh[c0:c1], v[c0:c1]
        G = np.cumsum(la[c0:c1])
        bb = b[c0:c1]
        n = c1 - c0
        D = np.exp(G[:, None] - G[None, :])
        A = np.tril(bb[:, None] * D * (K @ K.T), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ ((bb * np.exp(G))[:, None] * K)
        U = Tm @ (bb[:, None] * V)
        Delta = U - W @ S
        P = np.tril((Q @ K.T) * D)
        ys[c0:c1] = np.exp(G)[:, None] * (Q @ S) + P @ Delta
        S = np.exp(G[-1]) * S + (np.exp(G[-1] - G)[:, None] * K).T @ Delta
    return ys, S


@pytest.mark.parametrize("T,C", [(64, 16), (100, 32), (130, 64), (7, 64)])
def test_chunked_form_matches_recurrence(T, C):
    r = np.random.default_rng(T + C)
    dk, dv = 16, 12
    q = r.standard_normal((T, 1, dk)).astype(np.float32)
    k = r.standard_normal((T, 1, dk)).astype(np.float32)
    v = r.standard_normal((T, 1, dv)).astype(np.float32)
    la = (-np.log1p(np.exp(r.standard_normal((T, 1)))) * 0.5).astype(np.float32)
    b = (1 / (1 + np.exp(-r.standard_normal((T, 1))))).astype(np.float32)
    S0 = (r.standard_normal((1, 1, dk, dv)) * 0.3).astype(np.float32)
    y, fs = oracle.recurrence(q, k, v, la, b, initial_state=S0, eps_l2=0.0)
    unit = lambda x: x / np.sqrt((x * x).sum(-1, keepdims=True))
    yc, Sc = _chunked(unit(q[:, 0].astype(np.float64)), unit(k[:, 0].astype(np.float64)),
                      v[:, 0].astype(np.float64), la[:, 0].astype(np.float64),
                      b[:, 0].astype(np.float64), S0[0, 0].astype(np.float64), C)
    np.testing.assert_allclose(yc, y[:, 0], rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(Sc, fs[0, 0], rtol=1e-10, atol=1e-11)
