"""Multi-token decode (gdn_decode_multi) on the GPU: T_s tokens per sequence
in one launch with the state held on chip, optional per-token snapshots.

It must equal T_s single-token steps bit for bit (same arithmetic, the state
only stays in registers instead of going through memory), match the fp64
oracle, and its snapshots must be the states after each token (a caller rolls
back to an accepted prefix by taking one of them)."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_scan_chunked_b200 import gdn, gdn_decode_multi, gdn_decode_step, inputs
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _multi_inputs(d):
    """[steps, N, ...] decode inputs as the [N, T_s, ...] layout on the GPU."""
    tr = lambda x: None if x is None else x.transpose(0, 1).contiguous().cuda()
    return dict(q=tr(d.q), k=tr(d.k), v=tr(d.v), log_alpha=tr(d.log_alpha), beta=tr(d.beta),
                g=tr(d.g), norm_w=None if d.norm_w is None else d.norm_w.cuda())


def _single_steps(d, steps):
    state = d.state.clone().cuda()
    ys, states = [], []
    for t in range(steps):
        y = gdn_decode_step(d.q[t].cuda(), d.k[t].cuda(), d.v[t].cuda(),
                            d.log_alpha[t].cuda(), d.beta[t].cuda(), state,
                            g=None if d.g is None else d.g[t].cuda(),
                            norm_w=None if d.norm_w is None else d.norm_w.cuda())
        ys.append(y)
        states.append(state.clone())
    torch.cuda.synchronize()
    return torch.stack(ys, 1), states


def _oracle(d, n, heads, steps):
    Hqk, Hv = d.q.shape[2], d.v.shape[2]
    hq = [h // (Hv // Hqk) for h in heads]
    cpu = lambda x: x.to("cpu", torch.float32)
    return oracle.recurrence(
        cpu(d.q[:steps, n][:, hq]), cpu(d.k[:steps, n][:, hq]), cpu(d.v[:steps, n][:, heads]),
        cpu(d.log_alpha[:steps, n][:, heads]), cpu(d.beta[:steps, n][:, heads]),
        g=None if d.g is None else cpu(d.g[:steps, n][:, heads]),
        norm_w=None if d.norm_w is None else cpu(d.norm_w),
        initial_state=cpu(d.state[n][heads])[None])


@pytest.mark.parametrize("epilogue", [False, True])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_multi_equals_single_steps_bitwise(dtype, epilogue):
    d = inputs.make_decode(N=8, steps=6, dtype=dtype, epilogue=epilogue, seed=41)
    ys1, states1 = _single_steps(d, 6)
    m = _multi_inputs(d)
    state = d.state.clone().cuda()
    y, _ = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], state,
                            g=m["g"], norm_w=m["norm_w"])
    torch.cuda.synchronize()
    assert gdn.gdn_check_device_error() == gdn.GDN_OK
    assert torch.equal(y, ys1)
    assert torch.equal(state, states1[-1])


@pytest.mark.parametrize("dtype,epilogue", [(torch.bfloat16, True), (torch.float32, False)])
def test_multi_vs_oracle(dtype, epilogue):
    d = inputs.make_decode(N=4, steps=4, dtype=dtype, epilogue=epilogue, seed=42)
    m = _multi_inputs(d)
    state = d.state.clone().cuda()
    y, _ = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], state,
                            g=m["g"], norm_w=m["norm_w"])
    torch.cuda.synchronize()
    for n in range(4):
        y_ref, s_ref = _oracle(d, n, list(range(48)), 4)
        assert_close(y[n], y_ref, dtype, "y seq %d" % n)
        assert_close(state[n], s_ref[0], dtype, "state seq %d" % n)


def test_snapshots_and_rollback():
    """Snapshot t = state after token t; state_in untouched when state_out is
    separate; decoding on from a snapshot equals decoding the accepted prefix."""
    d = inputs.make_decode(N=5, steps=4, epilogue=True, seed=43)
    ys1, states1 = _single_steps(d, 4)
    m = _multi_inputs(d)
    s_in = d.state.clone().cuda()
    s_out = torch.empty_like(s_in)
    y, snaps = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], s_in,
                                state_out=s_out, snapshots=True, g=m["g"], norm_w=m["norm_w"])
    torch.cuda.synchronize()
    assert torch.equal(s_in, d.state.cuda())
    assert torch.equal(s_out, states1[-1])
    for t in range(4):
        assert torch.equal(snaps[t], states1[t]), "snapshot %d" % t
    assert torch.equal(y, ys1)
    # accept 2 tokens: continue from snapshot 1 with token 2 == single-step path
    s_roll = snaps[1].clone()
    y2 = gdn_decode_step(d.q[2].cuda(), d.k[2].cuda(), d.v[2].cuda(), d.log_alpha[2].cuda(),
                         d.beta[2].cuda(), s_roll, g=d.g[2].cuda(), norm_w=d.norm_w.cuda())
    torch.cuda.synchronize()
    assert torch.equal(y2, ys1[:, 2]) and torch.equal(s_roll, states1[2])


def test_state_not_written_when_out_is_none():
    d = inputs.make_decode(N=3, steps=3, seed=44)
    m = _multi_inputs(d)
    s_in = d.state.clone().cuda()
    y, _ = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], s_in,
                            state_out=None)
    torch.cuda.synchronize()
    assert torch.equal(s_in, d.state.cuda())
    ys1, _ = _single_steps(d, 3)
    assert torch.equal(y, ys1)


def test_multi_full_batch_sampled():
    """256 sequences x 48 heads, 4 speculative tokens, in place; sampled
    (sequence, head) pairs against the oracle."""
    d = inputs.make_decode(steps=4, device="cuda", seed=45)
    m = _multi_inputs(d)
    state = d.state.clone()
    y, _ = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], state)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    for n in rng.choice(256, size=5, replace=False):
        heads = sorted(rng.choice(48, size=4, replace=False).tolist())
        y_ref, s_ref = _oracle(d, int(n), heads, 4)
        assert_close(y[n][:, heads], y_ref, torch.bfloat16, "y seq %d" % n)
        assert_close(state[n][heads], s_ref[0], torch.bfloat16, "state seq %d" % n)


@pytest.mark.parametrize("T_s", [1, 7, 32])
def test_multi_token_counts(T_s):
    """1 token (the loop kernel with a separate output state), an odd count,
    and the maximum of 32 tokens, against single steps."""
    d = inputs.make_decode(N=3, steps=T_s, epilogue=True, seed=46 + T_s)
    ys1, states1 = _single_steps(d, T_s)
    m = _multi_inputs(d)
    s_in = d.state.clone().cuda()
    s_out = torch.empty_like(s_in)
    y, _ = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], s_in,
                            state_out=s_out, g=m["g"], norm_w=m["norm_w"])
    torch.cuda.synchronize()
    assert gdn.gdn_check_device_error() == gdn.GDN_OK
    assert torch.equal(y, ys1) and torch.equal(s_out, states1[-1])


@pytest.mark.parametrize("dk,dv", [(16, 16), (128, 16), (16, 128), (64, 32)])
def test_multi_other_head_dims_fp32(dk, dv):
    d = inputs.make_decode(N=3, steps=5, H_qk=2, H_v=4, d_k=dk, d_v=dv, dtype=torch.float32,
                           epilogue=True, seed=dk + dv)
    ys1, states1 = _single_steps(d, 5)
    m = _multi_inputs(d)
    state = d.state.clone().cuda()
    y, _ = gdn_decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], state,
                            g=m["g"], norm_w=m["norm_w"])
    torch.cuda.synchronize()
    assert torch.equal(y, ys1) and torch.equal(state, states1[-1])
