"""Pins for the fp64 oracle, independent of the oracle itself.

Each test checks the oracle against something the pages or the mathematics
fix, chosen so that a plausible slip in the oracle (a dropped decay, a sign,
a transposed state, reading y before the update, a wrong head mapping, state
leaking across packed sequences, a mis-ordered epilogue) fails at least one:

* hand-worked example (tests/golden/hand_worked_d2.json), error form from
  "Qwen3.8-Flash-Next: architecture, efficiency and technical lineage",
  section 03 "Gated DeltaNet";
* P1  beta = 0: pure decay, closed form exp(sum log alpha) S0;
* P2  alpha = beta = 1 with orthonormal keys: exact retrieval of the values
      written, and overwrite of a key keeps only the last value (the
      "Error e" / "Write beta" boxes of section 03);
* P3  error form == product form alpha (I - beta k k^T) S + beta k v^T
      ("On the Design of Qwen3.8-Next Architecture ... close reading",
      section 4.1) == brute-force product of dense transition matrices;
* P4  alpha = 1, beta = 0: y_t = S0^T q_t;
* P5  splitting a sequence and carrying the state == one pass;
* P6  spectral-norm bound of every step for unit keys and beta in (0,1);
* P7  packed sequences == each sequence alone; no leakage;
* P8  epilogue: rms of the output is (1+c) * sigmoid(g) for w = c;
      output is invariant to a joint scaling of v and S0;
* L2 norm: invariance of every output to positive rescaling of q and k;
* head grouping: value head h reads QK head h // (H_v / H_qk).
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_seed = 12345


def _rand_case(T, Hqk, Hv, dk, dv, seed, s0=True, n_seq_lengths=None, g=False):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, Hqk, dk)).astype(np.float32)
    k = r.standard_normal((T, Hqk, dk)).astype(np.float32)
    v = r.standard_normal((T, Hv, dv)).astype(np.float32)
    la = (-np.log1p(np.exp(r.standard_normal((T, Hv)))) * 0.3).astype(np.float32)
    b = (1 / (1 + np.exp(-r.standard_normal((T, Hv))))).astype(np.float32)
    lengths = n_seq_lengths or [T]
    S0 = (r.standard_normal((len(lengths), Hv, dk, dv)) * 0.1).astype(np.float32) if s0 else None
    gg = r.standard_normal((T, Hv, dv)).astype(np.float32) if g else None
    w = (r.standard_normal(dv) * 0.1).astype(np.float32) if g else None
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, g=gg, norm_w=w,
                initial_state=S0, cu_seqlens=cu)


def _unit(x):
    x = np.asarray(x, np.float64)
    return x / np.sqrt((x * x).sum(-1, keepdims=True))


def test_hand_worked_example():
    d = json.load(open(os.path.join(GOLDEN, "hand_worked_d2.json")))
    inp, exp = d["inputs"], d["expected"]
    q = np.array(inp["q"], np.float32)[:, None, :]
    k = np.array(inp["k"], np.float32)[:, None, :]
    v = np.array(inp["v"], np.float32)[:, None, :]
    la = np.log(np.array(inp["alpha"], np.float64)).astype(np.float32)[:, None]
    b = np.array(inp["beta"], np.float32)[:, None]
    s0 = np.array(inp["s0"], np.float32)[None, None]
    y, fs = oracle.recurrence(q, k, v, la, b, initial_state=s0, l2norm=False)
    np.testing.assert_allclose(y[:, 0], exp["y"], rtol=0, atol=1e-6)
    np.testing.assert_allclose(fs[0, 0], exp["final_state"], rtol=0, atol=1e-6)
    g = np.array(inp["g"], np.float32)[:, None, :]
    w = np.array(inp["norm_w"], np.float32)
    ye, _ = oracle.recurrence(q, k, v, la, b, g=g, norm_w=w, initial_state=s0,
                              l2norm=False, eps_norm=0.0)
    np.testing.assert_allclose(ye[:, 0], exp["y_epilogue"], rtol=0, atol=1e-6)


def test_p1_beta_zero_is_pure_decay():
    c = _rand_case(40, 1, 1, 8, 6, 1)
    c["beta"][:] = 0.0
    y, fs = oracle.recurrence(**c, eps_l2=0.0)
    S0 = c["initial_state"][0, 0].astype(np.float64)
    G = np.cumsum(c["log_alpha"][:, 0].astype(np.float64))
    np.testing.assert_allclose(fs[0, 0], np.exp(G[-1]) * S0, rtol=1e-12, atol=1e-15)
    qh = _unit(c["q"][:, 0])
    expect_y = np.exp(G)[:, None] * (qh @ S0)
    np.testing.assert_allclose(y[:, 0], expect_y, rtol=1e-11, atol=1e-14)


def test_p2_orthonormal_retrieval_and_overwrite():
    dk = dv = 8
    r = np.random.default_rng(2)
    Qm, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    keys = Qm.T  # rows orthonormal
    T = dk
    v = r.standard_normal((T, dv))
    # store fp64-exact fp32 values: use keys already rounded to fp32 and
    # compare with a tolerance covering fp32 rounding of the unit keys
    k32 = keys.astype(np.float32)
    q32 = k32.copy()
    y, fs = oracle.recurrence(q32[:, None], k32[:, None], v.astype(np.float32)[:, None],
                              np.zeros((T, 1), np.float32), np.ones((T, 1), np.float32),
                              l2norm=True, eps_l2=0.0)
    kh = _unit(k32)
    S = fs[0, 0]
    # every written key retrieves its value: S^T k_i = v_i
    np.testing.assert_allclose(kh @ S, v.astype(np.float32), atol=1e-5)
    # y_t reads the state after token t is written: y_t = v_t
    np.testing.assert_allclose(y[:, 0], v.astype(np.float32), atol=1e-5)
    # overwrite: same key twice, the later value wins
    kk = np.stack([k32[0], k32[0]])
    vv = np.stack([v[0], v[1]]).astype(np.float32)
    y2, fs2 = oracle.recurrence(kk[:, None], kk[:, None], vv[:, None],
                                np.zeros((2, 1), np.float32), np.ones((2, 1), np.float32),
                                l2norm=True, eps_l2=0.0)
    np.testing.assert_allclose(_unit(k32[0]) @ fs2[0, 0], vv[1], atol=1e-5)
    np.testing.assert_allclose(y2[1, 0], vv[1], atol=1e-5)


def _brute_force(qh, kh, v, alpha, beta, S0):
    """S_T = F_T..F_1 S0 + sum_t F_T..F_{t+1} beta_t k_t v_t^T with
    F_t = alpha_t (I - beta_t k_t k_t^T), every product formed densely."""
    T, dk = kh.shape
    F = [alpha[t] * (np.eye(dk) - beta[t] * np.outer(kh[t], kh[t])) for t in range(T)]
    ys = []
    for t_end in range(1, T + 1):
        P = np.eye(dk)
        S = np.zeros((dk, v.shape[1]))
        for t in range(t_end):
            # contribution of the write at t, carried through F_{t+1..t_end-1}
            P_after = np.eye(dk)
            for s in range(t + 1, t_end):
                P_after = F[s] @ P_after
            S += P_after @ (beta[t] * np.outer(kh[t], v[t]))
            P = F[t] @ P
        S += P @ S0
        ys.append(S.T @ qh[t_end - 1])
    return np.array(ys), S


@pytest.mark.parametrize("dk,dv,T", [(4, 6, 12), (16, 16, 32), (6, 3, 20)])
def test_p3_error_form_equals_product_form_and_brute_force(dk, dv, T):
    c = _rand_case(T, 1, 1, dk, dv, 3 + dk)
    y, fs = oracle.recurrence(**c, eps_l2=0.0)
    qh, kh = _unit(c["q"][:, 0]), _unit(c["k"][:, 0])
    v = c["v"][:, 0].astype(np.float64)
    a = np.exp(c["log_alpha"][:, 0].astype(np.float64))
    b = c["beta"][:, 0].astype(np.float64)
    S0 = c["initial_state"][0, 0].astype(np.float64)
    yp, sp = oracle.product_form(qh, kh, v, a, b, S0)
    np.testing.assert_allclose(y[:, 0], yp, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], sp, rtol=1e-12, atol=1e-12)
    yb, sb = _brute_force(qh, kh, v, a, b, S0)
    np.testing.assert_allclose(y[:, 0], yb, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], sb, rtol=1e-11, atol=1e-12)


def test_p4_no_write_no_decay_reads_initial_state():
    c = _rand_case(30, 2, 4, 8, 8, 4)
    c["beta"][:] = 0.0
    c["log_alpha"][:] = 0.0
    y, fs = oracle.recurrence(**c, eps_l2=0.0)
    for h in range(4):
        qh = _unit(c["q"][:, h // 2])
        S0 = c["initial_state"][0, h].astype(np.float64)
        np.testing.assert_allclose(y[:, h], qh @ S0, rtol=1e-12, atol=1e-14)
        np.testing.assert_array_equal(fs[0, h], S0)


def test_p5_split_and_carry_equals_one_pass():
    c = _rand_case(50, 1, 3, 8, 8, 5, g=True)
    y, fs = oracle.recurrence(**c)
    t1 = 23
    a = {kk: (vv[:t1] if (vv is not None and kk in ("q", "k", "v", "log_alpha", "beta", "g")) else vv)
         for kk, vv in c.items()}
    a["cu_seqlens"] = np.array([0, t1])
    ya, fa = oracle.recurrence(**a)
    b = {kk: (vv[t1:] if (vv is not None and kk in ("q", "k", "v", "log_alpha", "beta", "g")) else vv)
         for kk, vv in c.items()}
    b["cu_seqlens"] = np.array([0, 50 - t1])
    # the carried fp64 state, passed back in: it must be fp32 for the C
    # interface, so compare the second half against a pass resumed from the
    # fp32-rounded state with the appropriate tolerance, and the first half
    # bit for bit
    b["initial_state"] = fa.astype(np.float32)
    yb, fb = oracle.recurrence(**b)
    np.testing.assert_array_equal(ya, y[:t1])
    np.testing.assert_allclose(yb, y[t1:], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(fb, fs, rtol=1e-5, atol=1e-6)


def test_p6_norm_bound_each_step():
    c = _rand_case(24, 1, 1, 8, 8, 6)
    S = c["initial_state"][0, 0].astype(np.float64)
    s_prev = np.linalg.norm(S, 2)
    Sin = c["initial_state"]
    for t in range(24):
        one = {kk: (vv[t:t + 1] if (vv is not None and kk in ("q", "k", "v", "log_alpha", "beta")) else vv)
               for kk, vv in c.items()}
        one["cu_seqlens"] = np.array([0, 1])
        one["initial_state"] = Sin
        _, fs = oracle.recurrence(**one)
        s_now = np.linalg.norm(fs[0, 0], 2)
        bound = np.exp(float(c["log_alpha"][t, 0])) * np.linalg.norm(Sin[0, 0].astype(np.float64), 2) \
            + float(c["beta"][t, 0]) * np.linalg.norm(c["v"][t, 0].astype(np.float64))
        assert s_now <= bound * (1 + 1e-12) + 1e-12
        Sin = fs.astype(np.float32)
    del s_prev


def test_p7_packing_equals_separate_runs_and_no_leakage():
    lengths = [7, 0, 19, 1, 33]
    c = _rand_case(sum(lengths), 2, 4, 8, 8, 7, n_seq_lengths=lengths, g=True)
    y, fs = oracle.recurrence(**c)
    cu = c["cu_seqlens"]
    for s, L in enumerate(lengths):
        t0, t1 = cu[s], cu[s + 1]
        one = {kk: (vv[t0:t1] if (vv is not None and kk in ("q", "k", "v", "log_alpha", "beta", "g")) else vv)
               for kk, vv in c.items()}
        one["cu_seqlens"] = np.array([0, L])
        one["initial_state"] = c["initial_state"][s:s + 1]
        ys, fss = oracle.recurrence(**one)
        np.testing.assert_array_equal(ys, y[t0:t1])
        np.testing.assert_array_equal(fss[0], fs[s])
    # empty sequence: final state = initial state
    np.testing.assert_array_equal(fs[1], c["initial_state"][1].astype(np.float64))
    # perturb sequence 2 only: others unchanged
    c2 = {kk: (vv.copy() if isinstance(vv, np.ndarray) else vv) for kk, vv in c.items()}
    c2["v"][cu[2]:cu[3]] += 1.0
    y2, fs2 = oracle.recurrence(**c2)
    for s in (0, 1, 3, 4):
        np.testing.assert_array_equal(y2[cu[s]:cu[s + 1]], y[cu[s]:cu[s + 1]])
        np.testing.assert_array_equal(fs2[s], fs[s])
    assert np.abs(y2[cu[2]:cu[3]] - y[cu[2]:cu[3]]).max() > 1e-3


def test_p8_epilogue_rms_and_gate():
    c = _rand_case(16, 1, 2, 8, 8, 8, g=True)
    # w = c0 constant, g -> +inf: rms(out) == 1 + c0
    c["g"][:] = 40.0
    c["norm_w"][:] = 0.25
    y, _ = oracle.recurrence(**c, eps_norm=0.0)
    rms = np.sqrt((y ** 2).mean(-1))
    np.testing.assert_allclose(rms, 1.25, rtol=1e-12)
    # g = 0: exactly half of that
    c["g"][:] = 0.0
    y0, _ = oracle.recurrence(**c, eps_norm=0.0)
    np.testing.assert_allclose(np.sqrt((y0 ** 2).mean(-1)), 0.625, rtol=1e-12)
    np.testing.assert_allclose(y0, 0.5 * y, rtol=1e-12, atol=1e-15)
    # direction of each head output is that of the raw y (normalise, then gate)
    c_raw = dict(c)
    c_raw["g"] = None
    c_raw["norm_w"] = None
    yr, _ = oracle.recurrence(**c_raw)
    cos = (y * yr).sum(-1) / np.linalg.norm(y, axis=-1) / np.linalg.norm(yr, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-12)
    # joint scaling of v and S0 leaves the epilogue output unchanged
    c3 = {kk: (vv.copy() if isinstance(vv, np.ndarray) else vv) for kk, vv in c.items()}
    c3["g"] = np.random.default_rng(1).standard_normal(c["g"].shape).astype(np.float32)
    y3, _ = oracle.recurrence(**c3, eps_norm=0.0)
    c3["v"] = c3["v"] * 4.0
    c3["initial_state"] = c3["initial_state"] * 4.0
    y4, _ = oracle.recurrence(**c3, eps_norm=0.0)
    np.testing.assert_allclose(y4, y3, rtol=1e-12, atol=1e-14)


def test_l2norm_invariance_and_scale_linearity():
    c = _rand_case(20, 2, 4, 8, 8, 9)
    y, fs = oracle.recurrence(**c, eps_l2=0.0)
    c2 = dict(c)
    c2["q"] = c["q"] * 4.0
    c2["k"] = c["k"] * 0.25
    y2, fs2 = oracle.recurrence(**c2, eps_l2=0.0)
    np.testing.assert_allclose(y2, y, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(fs2, fs, rtol=1e-10, atol=1e-12)
    # without normalisation the raw scaling shows up
    y3, _ = oracle.recurrence(**c2, l2norm=False)
    assert np.abs(y3 - y).max() > 1e-2
    # scale multiplies y and leaves the state alone
    y5, fs5 = oracle.recurrence(**c, eps_l2=0.0, scale=0.125)
    np.testing.assert_allclose(y5, 0.125 * y, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(fs5, fs)


def test_head_grouping_is_contiguous():
    Hqk, Hv = 2, 6
    c = _rand_case(15, Hqk, Hv, 8, 8, 10, g=True)
    y, fs = oracle.recurrence(**c)
    G = Hv // Hqk
    for h in range(Hv):
        one = dict(c)
        one["q"] = c["q"][:, h // G:h // G + 1]
        one["k"] = c["k"][:, h // G:h // G + 1]
        for kk in ("v", "log_alpha", "beta", "g"):
            one[kk] = c[kk][:, h:h + 1]
        one["initial_state"] = c["initial_state"][:, h:h + 1]
        ys, fss = oracle.recurrence(**one)
        np.testing.assert_array_equal(ys[:, 0], y[:, h])
        np.testing.assert_array_equal(fss[:, 0], fs[:, h])


def test_rejects_bad_arguments():
    c = _rand_case(10, 2, 4, 8, 8, 11)
    c["cu_seqlens"] = np.array([0, 6, 4, 10])
    with pytest.raises(ValueError):
        oracle.recurrence(**c)
    c["cu_seqlens"] = np.array([0, 11])
    with pytest.raises(ValueError):
        oracle.recurrence(**c)
