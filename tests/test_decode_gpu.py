"""Decode step on the GPU against the fp64 oracle.

The oracle runs the same tokens as a prefill of one token per step from the
same state (the recurrence is the same; the decode kernel's closed form
y = alpha S^T q + beta (k.q) e is only an algebraic regrouping of it).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_scan_chunked_b200 import gdn_decode_step, inputs
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _oracle_steps(d, n, heads, steps, **kw):
    """Oracle for sequence n over `steps` tokens, value heads `heads`."""
    Hqk, Hv = d.q.shape[2], d.v.shape[2]
    G = Hv // Hqk
    hq = [h // G for h in heads]
    cpu = lambda x: x.to("cpu", torch.float32)
    q = cpu(d.q[:steps, n][:, hq])
    k = cpu(d.k[:steps, n][:, hq])
    v = cpu(d.v[:steps, n][:, heads])
    la = cpu(d.log_alpha[:steps, n][:, heads])
    b = cpu(d.beta[:steps, n][:, heads])
    g = None if d.g is None else cpu(d.g[:steps, n][:, heads])
    w = None if d.norm_w is None else cpu(d.norm_w)
    s0 = cpu(d.state[n][heads])[None]
    return oracle.recurrence(q, k, v, la, b, g=g, norm_w=w, initial_state=s0, **kw)


def _run(d, steps):
    state = d.state.clone().cuda()
    ys = []
    for t in range(steps):
        y = gdn_decode_step(d.q[t].cuda(), d.k[t].cuda(), d.v[t].cuda(),
                            d.log_alpha[t].cuda(), d.beta[t].cuda(), state,
                            g=None if d.g is None else d.g[t].cuda(),
                            norm_w=None if d.norm_w is None else d.norm_w.cuda())
        ys.append(y)
    torch.cuda.synchronize()
    return torch.stack(ys), state


@pytest.mark.parametrize("dtype,epilogue", [(torch.bfloat16, False), (torch.bfloat16, True),
                                            (torch.float32, False), (torch.float32, True)])
def test_decode_model_shape_small_batch(dtype, epilogue):
    d = inputs.make_decode(N=4, steps=64, dtype=dtype, epilogue=epilogue)
    ys, state = _run(d, 64)
    for n in range(4):
        y_ref, s_ref = _oracle_steps(d, n, list(range(48)), 64)
        assert_close(ys[:, n], y_ref, dtype, "y seq %d" % n)
        assert_close(state[n], s_ref[0], dtype, "state seq %d" % n)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 128), (128, 16), (64, 64), (16, 64)])
def test_decode_other_head_dims_fp32(dk, dv):
    d = inputs.make_decode(N=3, steps=20, H_qk=2, H_v=4, d_k=dk, d_v=dv, dtype=torch.float32,
                           epilogue=True)
    ys, state = _run(d, 20)
    for n in range(3):
        y_ref, s_ref = _oracle_steps(d, n, list(range(4)), 20)
        assert_close(ys[:, n], y_ref, torch.float32, "y")
        assert_close(state[n], s_ref[0], torch.float32, "state")


def test_decode_full_batch_sampled():
    """256 sequences x 48 heads, 64 steps (the batched-decode workload);
    the oracle checks sampled (sequence, head) pairs at every step."""
    d = inputs.make_decode(device="cuda")
    ys, state = _run(d, 64)
    rng = np.random.default_rng(0)
    for n in rng.choice(256, size=6, replace=False):
        heads = sorted(rng.choice(48, size=4, replace=False).tolist())
        y_ref, s_ref = _oracle_steps(d, int(n), heads, 64)
        assert_close(ys[:, n][:, heads], y_ref, torch.bfloat16, "y seq %d" % n)
        assert_close(state[n][heads], s_ref[0], torch.bfloat16, "state seq %d" % n)


def test_decode_matches_prefill_on_same_tokens():
    """64 decode steps == one 64-token prefill from the same state (GPU vs GPU)."""
    from gated_deltanet_scan_chunked_b200 import gdn_chunk_fwd
    d = inputs.make_decode(N=2, steps=64, epilogue=True)
    ys, state = _run(d, 64)
    for n in range(2):
        y, fs = gdn_chunk_fwd(d.q[:, n].contiguous().cuda(), d.k[:, n].contiguous().cuda(),
                              d.v[:, n].contiguous().cuda(),
                              d.log_alpha[:, n].contiguous().cuda(),
                              d.beta[:, n].contiguous().cuda(),
                              g=d.g[:, n].contiguous().cuda(), norm_w=d.norm_w.cuda(),
                              initial_state=d.state[n:n + 1].cuda())
        torch.cuda.synchronize()
        assert_close(y, ys[:, n].to(torch.float64).cpu().numpy(), torch.bfloat16, "y")
        assert_close(fs[0], state[n].cpu().numpy(), torch.bfloat16, "state")
