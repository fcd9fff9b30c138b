"""The chunkwise backward used by the CUDA backward kernels, checked in fp64
against the oracle's token-by-token adjoint.

Forward within a chunk (entering state S0, C tokens; see
test_chunked_derivation.py for the forward form), with Qs = scale * Q^,
E_ti = exp(G_t - G_i), gamma = exp(G), b = exp(G_C - G):

  A = diag(beta) (K K^T o E)_strict   T = (I + A)^-1
  W = T diag(beta gamma) K            U = T diag(beta) V
  Delta = U - W S0                    P = (Qs K^T o E)_lower-incl
  Y  = diag(gamma) Qs S0 + P Delta    S1 = gamma_C S0 + (diag(b) K)^T Delta

Backward, given dY and dS1 (the gradient of the state leaving the chunk):

  chain (d_v columns independent):
    dDelta = P^T dY + diag(b) K dS1
    dS0    = (diag(gamma) Qs)^T dY + gamma_C dS1 - W^T dDelta
  per chunk:
    TdD = T^T dDelta          dV = diag(beta) TdD
    R   = (I + A) Delta       (= diag(beta)(V - diag(gamma) K S0))
    dT  = dDelta R^T          dA = -(T^T dT T^T)_strict
    dP  = (dY Delta^T)_lower-incl
    L1 = dY S0^T   L2 = TdD S0^T   L3 = Delta dS1^T
    dQs = diag(gamma) L1 + (dP o E) K
    dK  = (dP o E)^T Qs + diag(b) L3 - diag(beta gamma) L2
          + (B + B^T) K,   B = dA o E o beta_t (strictly lower)
    dbeta_t = (TdD V^T)_tt - gamma_t (K L2^T)_tt + sum_i dA_ti (K K^T o E)_ti
    dG_t = sum_i (dP o P)_ti - sum_i (dP o P)_it + sum_i (dA o A)_ti - sum_i (dA o A)_it
           + gamma_t (Qs L1^T)_tt - beta_t gamma_t (K L2^T)_tt - b_t (K L3^T)_tt
    dG_last += sum_t b_t (K L3^T)_tt + gamma_C <S0, dS1>
    dlog_alpha = reverse cumulative sum of dG within the chunk
"""
import numpy as np
import pytest

import oracle


def _chunked_backward(qh, kh, v, la, b, S0, dY, dST, C, scale):
    T_, dk = kh.shape
    dv = v.shape[1]
    chunks = [(c0, min(T_, c0 + C)) for c0 in range(0, T_, C)]
    pre = []
    for c0, c1 in chunks:                      # per-chunk preparation
        K, Qs, V = kh[c0:c1], scale * qh[c0:c1], v[c0:c1]
        G = np.cumsum(la[c0:c1])
        bb = b[c0:c1]
        n = c1 - c0
        E = np.exp(G[:, None] - G[None, :])
        KKE = np.tril(K @ K.T * E, -1)
        A = bb[:, None] * KKE
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ ((bb * np.exp(G))[:, None] * K)
        U = Tm @ (bb[:, None] * V)
        P = np.tril(Qs @ K.T * E)
        pre.append(dict(K=K, Qs=Qs, V=V, G=G, b=bb, E=E, KKE=KKE, A=A, T=Tm, W=W, U=U, P=P))
    # forward chain: the state entering each chunk, and Delta
    S = S0.copy()
    for p in pre:
        p["S0"] = S.copy()
        p["D"] = p["U"] - p["W"] @ S
        bdec = np.exp(p["G"][-1] - p["G"])
        S = np.exp(p["G"][-1]) * S + (bdec[:, None] * p["K"]).T @ p["D"]
    # backward chain: dS1 of each chunk, and dDelta
    dS = dST.copy()
    for (c0, c1), p in reversed(list(zip(chunks, pre))):
        p["dS1"] = dS.copy()
        dYc = dY[c0:c1]
        bdec = np.exp(p["G"][-1] - p["G"])
        p["dD"] = p["P"].T @ dYc + (bdec[:, None] * p["K"]) @ dS
        dS = (np.exp(p["G"])[:, None] * p["Qs"]).T @ dYc + np.exp(p["G"][-1]) * dS \
            - p["W"].T @ p["dD"]
    dS0 = dS
    dq = np.zeros((T_, dk))
    dk_ = np.zeros((T_, dk))
    dv_ = np.zeros((T_, dv))
    dla = np.zeros(T_)
    dbeta = np.zeros(T_)
    for (c0, c1), p in zip(chunks, pre):
        dYc = dY[c0:c1]
        K, Qs, V, E, bb, Tm = p["K"], p["Qs"], p["V"], p["E"], p["b"], p["T"]
        gam = np.exp(p["G"])
        bdec = np.exp(p["G"][-1] - p["G"])
        TdD = Tm.T @ p["dD"]
        dv_[c0:c1] = bb[:, None] * TdD
        R = p["D"] + p["A"] @ p["D"]
        dT = p["dD"] @ R.T
        dA = np.tril(-(Tm.T @ dT @ Tm.T), -1)
        dP = np.tril(dYc @ p["D"].T)
        L1 = dYc @ p["S0"].T
        L2 = TdD @ p["S0"].T
        L3 = p["D"] @ p["dS1"].T
        dPE = dP * E
        B = dA * E * bb[:, None]
        dQs = gam[:, None] * L1 + dPE @ K
        dK = dPE.T @ Qs + bdec[:, None] * L3 - (bb * gam)[:, None] * L2 + (B + B.T) @ K
        kl2 = (K * L2).sum(1)
        dbeta[c0:c1] = (TdD * V).sum(1) - gam * kl2 + (dA * p["KKE"]).sum(1)
        PP = dP * p["P"]
        AA = dA * p["A"]
        db = (K * L3).sum(1)
        dG = PP.sum(1) - PP.sum(0) + AA.sum(1) - AA.sum(0) + gam * (Qs * L1).sum(1) \
            - bb * gam * kl2 - bdec * db
        dG[-1] += (bdec * db).sum() + gam[-1] * (p["S0"] * p["dS1"]).sum()
        dla[c0:c1] = np.cumsum(dG[::-1])[::-1]
        dq[c0:c1] = scale * dQs
        dk_[c0:c1] = dK
    return dict(dqh=dq, dkh=dk_, dv=dv_, dlog_alpha=dla, dbeta=dbeta, d_initial_state=dS0)


@pytest.mark.parametrize("T,C,scale", [(64, 16, 1.0), (100, 32, 0.5), (130, 64, 1.0), (7, 64, 2.0)])
def test_chunked_backward_matches_adjoint(T, C, scale):
    r = np.random.default_rng(T + C)
    dk, dv = 16, 12
    q = r.standard_normal((T, 1, dk)).astype(np.float32)
    k = r.standard_normal((T, 1, dk)).astype(np.float32)
    v = r.standard_normal((T, 1, dv)).astype(np.float32)
    la = (-np.log1p(np.exp(r.standard_normal((T, 1)))) * 0.5).astype(np.float32)
    b = (1 / (1 + np.exp(-r.standard_normal((T, 1))))).astype(np.float32)
    S0 = (r.standard_normal((1, 1, dk, dv)) * 0.3).astype(np.float32)
    dy = r.standard_normal((T, 1, dv)).astype(np.float32)
    dST = r.standard_normal((1, 1, dk, dv)).astype(np.float32)
    # l2norm off: the chunked form acts on the normalised q, k the kernels use
    ref = oracle.backward(q, k, v, la, b, dy, initial_state=S0, d_final_state=dST,
                          l2norm=False, scale=scale)
    got = _chunked_backward(q[:, 0].astype(np.float64), k[:, 0].astype(np.float64),
                            v[:, 0].astype(np.float64), la[:, 0].astype(np.float64),
                            b[:, 0].astype(np.float64), S0[0, 0].astype(np.float64),
                            dy[:, 0].astype(np.float64), dST[0, 0].astype(np.float64), C, scale)
    for name, gname in [("dqh", "dq"), ("dkh", "dk"), ("dv", "dv"), ("dlog_alpha", "dlog_alpha"),
                        ("dbeta", "dbeta"), ("d_initial_state", "d_initial_state")]:
        want = ref[gname][:, 0] if gname != "d_initial_state" else ref[gname][0, 0]
        np.testing.assert_allclose(got[name], want, rtol=1e-9, atol=1e-10, err_msg=name)
