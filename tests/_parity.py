"""Helpers for comparing the CUDA path with the fp64 oracle.

Tolerances (the acceptance bar for this library):
  bf16 inputs: relative L2 error <= 1e-2 and max abs error <= 2e-2, on y and
               on the final state;
  fp32 inputs: relative L2 error <= 1e-4 (and max abs error <= 1e-3 as a
               guard against isolated spikes).
"""
import numpy as np
import torch

import oracle

TOL = {
    torch.bfloat16: dict(rel_l2=1e-2, max_abs=2e-2),
    torch.float32: dict(rel_l2=1e-4, max_abs=1e-3),
}


def errors(got, ref):
    got = np.asarray(got.detach().to("cpu", torch.float64) if hasattr(got, "detach") else got,
                     dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if not np.isfinite(got).all():
        return float("inf"), float("inf")
    d = got - ref
    den = np.sqrt((ref * ref).sum())
    rel = float(np.sqrt((d * d).sum()) / den) if den > 0 else float(np.sqrt((d * d).sum()))
    return rel, float(np.abs(d).max()) if d.size else 0.0


def assert_close(got, ref, dtype, what=""):
    tol = TOL[dtype]
    rel, mx = errors(got, ref)
    assert rel <= tol["rel_l2"] and mx <= tol["max_abs"], (
        "%s: rel_l2=%.3e (tol %.0e) max_abs=%.3e (tol %.0e)"
        % (what, rel, tol["rel_l2"], mx, tol["max_abs"]))
    return rel, mx


def oracle_prefill(w, heads=None, seqs=None, n_threads=0, **kw):
    """Run the oracle on (a subset of) a PrefillInputs workload.

    heads: value heads to compute (None = all); seqs: sequence indices (None =
    all).  Returns (y [T_sel, len(heads), d_v], final [len(seqs), len(heads),
    d_k, d_v]) where T_sel are the tokens of the selected sequences, in order.
    """
    Hqk, Hv = w.q.shape[1], w.v.shape[1]
    G = Hv // Hqk
    heads = list(range(Hv)) if heads is None else list(heads)
    cu = w.cu_seqlens.to("cpu").numpy().astype(np.int64)
    seqs = list(range(len(cu) - 1)) if seqs is None else list(seqs)
    tok = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]) if seqs else \
        np.zeros(0, np.int64)
    lens = [int(cu[s + 1] - cu[s]) for s in seqs]
    sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ti = torch.as_tensor(tok, dtype=torch.long)
    hq = torch.as_tensor([h // G for h in heads], dtype=torch.long)
    hv = torch.as_tensor(heads, dtype=torch.long)

    def pick(x, hidx):
        if x is None:
            return None
        x = x.index_select(1, hidx.to(x.device)) if x.dim() >= 2 else x
        return x.index_select(0, ti.to(x.device)).to("cpu", torch.float32)

    s0 = None
    if w.initial_state is not None:
        s0 = w.initial_state.index_select(0, torch.as_tensor(seqs, dtype=torch.long,
                                                             device=w.initial_state.device))
        s0 = s0.index_select(1, hv.to(s0.device)).to("cpu", torch.float32)
    # each selected value head gets its own copy of its QK head: H_qk = H_v
    y, fs = oracle.recurrence(
        pick(w.q, hq), pick(w.k, hq), pick(w.v, hv), pick(w.log_alpha, hv),
        pick(w.beta, hv), g=pick(w.g, hv),
        norm_w=None if w.norm_w is None else w.norm_w.to("cpu", torch.float32),
        initial_state=s0, cu_seqlens=sub_cu, n_threads=n_threads, **kw)
    return y, fs, tok


def to_device(w, device="cuda"):
    """Copy every tensor of a PrefillInputs to the device."""
    import dataclasses
    out = {}
    for f in dataclasses.fields(w):
        x = getattr(w, f.name)
        out[f.name] = x.to(device) if isinstance(x, torch.Tensor) else x
    return type(w)(**out)
