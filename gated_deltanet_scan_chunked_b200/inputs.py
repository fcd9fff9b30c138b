"""Seeded synthetic inputs for the gated delta rule workloads.

This module draws random numbers and rounds them to the storage dtype; it
holds none of the method's arithmetic.  Both the CUDA path and the fp64
oracle consume exactly the tensors it returns (CPU tensors; callers move
them to the device), so the two sides see identical bf16-rounded values.

Workloads (head geometry from the GDN row of the module table in
"Qwen3.8-Flash-Next: architecture, efficiency and technical lineage",
section 02: 48 value heads share 16 QK heads, head dim 128):

* ``tiny``        T=64, H_qk=2, H_v=4, d=16, fp32; alpha = sigmoid(N(2,1));
                  zero initial state; no output epilogue.
* ``prefill4k``   T=4096, 16/48 heads, d=128, bf16 q/k/v/g; log alpha =
                  -softplus(N(0,1)) * 0.1; beta = sigmoid(N(0,1)); norm
                  weight N(0, 0.02^2); zero initial state.
* ``prefill256k`` as prefill4k with T=262,144 and initial state N(0, 0.01^2).
* ``varlen``      24 sequences, lengths uniform in [512, 16384], packed
                  with cu_seqlens, each with its own N(0, 0.01^2) state.
* ``decode``      256 sequences, state N(0, 0.05^2) [256, 48, 128, 128],
                  64 single-token steps of bf16 q/k/v and fp32 gates.

q and k are drawn N(0,1) and are L2-normalised by the consumer (the kernel's
prologue, or the oracle), as the workloads specify.

``device="cpu"`` (default) draws with torch's CPU generator; ``device="cuda"``
draws the same distributions with torch's CUDA (Philox) generator, which is
what the full-size workloads use (drawing 2.4 G normals on one CPU core takes
about a minute).  The two streams differ; a given (workload, device, seed)
is reproducible.  Oracle comparisons copy the sampled slices to the host.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

WORKLOADS = ("tiny", "prefill4k", "prefill256k", "varlen", "decode")
SEEDS = {name: 1000 + i for i, name in enumerate(WORKLOADS)}

# Random draws of big tensors are made in blocks of this many tokens so that
# the fp32 staging buffer stays small; the block size is part of the recipe.
_BLOCK_TOKENS = 8192


@dataclass
class PrefillInputs:
    q: torch.Tensor                 # [T, H_qk, d_k]   dtype
    k: torch.Tensor                 # [T, H_qk, d_k]   dtype
    v: torch.Tensor                 # [T, H_v, d_v]    dtype
    log_alpha: torch.Tensor         # [T, H_v]         fp32, <= 0
    beta: torch.Tensor              # [T, H_v]         fp32, in (0, 1)
    g: Optional[torch.Tensor]       # [T, H_v, d_v]    dtype, or None
    norm_w: Optional[torch.Tensor]  # [d_v]            fp32, or None
    initial_state: Optional[torch.Tensor]  # [n_seq, H_v, d_k, d_v] fp32 or None
    cu_seqlens: torch.Tensor        # [n_seq + 1]      int32
    meta: dict = field(default_factory=dict)

    @property
    def total_T(self) -> int:
        return int(self.q.shape[0])

    @property
    def n_seq(self) -> int:
        return int(self.cu_seqlens.shape[0]) - 1


@dataclass
class DecodeInputs:
    state: torch.Tensor             # [N, H_v, d_k, d_v] fp32
    q: torch.Tensor                 # [steps, N, H_qk, d_k] dtype
    k: torch.Tensor                 # [steps, N, H_qk, d_k] dtype
    v: torch.Tensor                 # [steps, N, H_v, d_v]  dtype
    log_alpha: torch.Tensor         # [steps, N, H_v] fp32
    beta: torch.Tensor              # [steps, N, H_v] fp32
    g: Optional[torch.Tensor] = None
    norm_w: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)


def _normal(gen, shape, dtype, std=1.0, mean=0.0):
    """N(mean, std^2) drawn in fp32 in token blocks, rounded to ``dtype``."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype, device=gen.device)
    if len(shape) == 0 or shape[0] == 0:
        return out
    rest = shape[1:]
    for t0 in range(0, shape[0], _BLOCK_TOKENS):
        t1 = min(shape[0], t0 + _BLOCK_TOKENS)
        x = torch.randn((t1 - t0,) + rest, generator=gen, dtype=torch.float32,
                        device=gen.device)
        if std != 1.0:
            x.mul_(std)
        if mean != 0.0:
            x.add_(mean)
        out[t0:t1] = x.to(dtype)
    return out


def _gates(gen, T, Hv, alpha_kind):
    if alpha_kind == "sigmoid_n2":
        # alpha = sigmoid(N(2,1)); stored as log(alpha)
        x = torch.randn((T, Hv), generator=gen, dtype=torch.float32, device=gen.device) + 2.0
        log_alpha = torch.nn.functional.logsigmoid(x)
    else:
        # log alpha = -softplus(N(0,1)) * 0.1
        x = torch.randn((T, Hv), generator=gen, dtype=torch.float32, device=gen.device)
        log_alpha = -torch.nn.functional.softplus(x) * 0.1
    beta = torch.sigmoid(torch.randn((T, Hv), generator=gen, dtype=torch.float32,
                                     device=gen.device))
    return log_alpha.contiguous(), beta.contiguous()


def _gen(seed, device):
    return torch.Generator(device=device).manual_seed(int(seed))


def make_prefill(lengths, H_qk, H_v, d_k, d_v, dtype=torch.bfloat16, seed=0,
                 epilogue=True, s0_std=0.0, alpha_kind="softplus01", device="cpu"):
    """Generic seeded prefill inputs over sequences of the given lengths."""
    gen = _gen(seed, device)
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    if lengths:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    cu = cu.to(device)
    q = _normal(gen, (T, H_qk, d_k), dtype)
    k = _normal(gen, (T, H_qk, d_k), dtype)
    v = _normal(gen, (T, H_v, d_v), dtype)
    log_alpha, beta = _gates(gen, T, H_v, alpha_kind)
    g = _normal(gen, (T, H_v, d_v), dtype) if epilogue else None
    norm_w = (torch.randn((d_v,), generator=gen, dtype=torch.float32, device=gen.device) * 0.02
              if epilogue else None)
    s0 = None
    if s0_std > 0.0:
        s0 = _normal(gen, (len(lengths), H_v, d_k, d_v), torch.float32, std=s0_std)
    return PrefillInputs(q, k, v, log_alpha, beta, g, norm_w, s0, cu,
                         meta={"lengths": lengths, "seed": int(seed)})


def make_cotangents(w: PrefillInputs, seed=0, ds_std=0.5, final_grad=True):
    """Seeded gradients for a backward pass over the prefill inputs ``w``:
    dy ~ N(0, 1) in the dtype of q (shape of y) and, if ``final_grad``,
    d_final_state ~ N(0, ds_std^2) fp32 [n_seq, H_v, d_k, d_v]."""
    gen = _gen(int(seed) + 99, w.q.device)
    T, Hv, dv = w.v.shape
    dk = w.q.shape[2]
    dy = _normal(gen, (T, Hv, dv), w.q.dtype)
    dsT = None
    if final_grad:
        dsT = _normal(gen, (w.cu_seqlens.shape[0] - 1, Hv, dk, dv), torch.float32, std=ds_std)
    return dy, dsT


def make_conv_params(n_seq, H_qk, H_v, d_k, d_v, seed=0, w_std=0.5, state=True,
                     device="cpu"):
    """Seeded front-end parameters: conv_w ~ N(0, w_std^2) fp32
    [2 H_qk d_k + H_v d_v, 4] and, if ``state``, a carried conv state
    ~ N(0, 1) fp32 [n_seq, H_v, 3, 2 d_k + d_v] whose q/k part is the same
    in every value head of a group (as the library keeps it)."""
    gen = _gen(int(seed) + 77, device)
    C = 2 * H_qk * d_k + H_v * d_v
    w = torch.randn((C, 4), generator=gen, dtype=torch.float32, device=device) * w_std
    st = None
    if state:
        G = H_v // H_qk
        qk = torch.randn((n_seq, H_qk, 3, 2 * d_k), generator=gen, dtype=torch.float32,
                         device=device)
        vv = torch.randn((n_seq, H_v, 3, d_v), generator=gen, dtype=torch.float32,
                         device=device)
        st = torch.cat([qk.repeat_interleave(G, dim=1), vv], dim=3).contiguous()
    return w, st


def make_gr(T, n_r=4, d=2560, rank=320, seed=0, device="cpu"):
    """Seeded Gated Residual inputs: an E4M3 state given directly as codes
    (random sign, exponent field 4..14, mantissa; no NaN codes) with fp32
    scales ~ U(0.01, 0.1), gains ~ 1 + N(0, 0.1^2), router and write weights
    ~ N(0, 1/fan_in) in bf16, a block output y ~ N(0, 1) bf16 and write
    scalars s ~ U(0.1, 1.9)."""
    gen = _gen(int(seed) + 500, device)
    sign = torch.randint(0, 2, (T, n_r, d), generator=gen, device=device)
    expo = torch.randint(4, 15, (T, n_r, d), generator=gen, device=device)
    mant = torch.randint(0, 8, (T, n_r, d), generator=gen, device=device)
    codes = (sign * 128 + expo * 8 + mant).to(torch.uint8)
    scales = torch.rand((T, n_r), generator=gen, device=device) * 0.09 + 0.01
    gamma = 1.0 + 0.1 * torch.randn((n_r, d), generator=gen, device=device)
    nd = n_r * d
    W_d = (torch.randn((rank, nd), generator=gen, device=device) / nd ** 0.5).to(torch.bfloat16)
    W_u = (torch.randn((nd, rank), generator=gen, device=device) / rank ** 0.5).to(torch.bfloat16)
    W_w = (torch.randn((n_r, nd), generator=gen, device=device) / nd ** 0.5).to(torch.bfloat16)
    y = torch.randn((T, d), generator=gen, device=device).to(torch.bfloat16)
    s = torch.rand((T, n_r), generator=gen, device=device) * 1.8 + 0.1
    return dict(codes=codes, scales=scales.float(), gamma=gamma.float(), W_d=W_d, W_u=W_u,
                W_w=W_w, y=y, s=s.float())


def varlen_lengths(n_seq=24, lo=512, hi=16384, seed=SEEDS["varlen"]):
    """Sequence lengths drawn uniformly from the integers [lo, hi]."""
    gen = torch.Generator().manual_seed(int(seed) + 7)
    return [int(x) for x in torch.randint(lo, hi + 1, (n_seq,), generator=gen)]


def workload(name: str, T: Optional[int] = None, device="cpu"):
    """The named workload's inputs.  ``T`` shortens a prefill workload
    (same recipe, fewer tokens) for oracle-sized parity cases."""
    seed = SEEDS[name]
    if name == "tiny":
        return make_prefill([T or 64], 2, 4, 16, 16, dtype=torch.float32,
                            seed=seed, epilogue=False, s0_std=0.0,
                            alpha_kind="sigmoid_n2", device=device)
    if name == "prefill4k":
        return make_prefill([T or 4096], 16, 48, 128, 128, seed=seed, device=device)
    if name == "prefill256k":
        return make_prefill([T or 262144], 16, 48, 128, 128, seed=seed, s0_std=0.01,
                            device=device)
    if name == "varlen":
        return make_prefill(varlen_lengths(), 16, 48, 128, 128, seed=seed, s0_std=0.01,
                            device=device)
    raise KeyError(name)


def make_decode(N=256, steps=64, H_qk=16, H_v=48, d_k=128, d_v=128,
                dtype=torch.bfloat16, seed=SEEDS["decode"], state_std=0.05,
                epilogue=False, device="cpu"):
    gen = _gen(seed, device)
    state = _normal(gen, (N, H_v, d_k, d_v), torch.float32, std=state_std)
    q = _normal(gen, (steps, N, H_qk, d_k), dtype)
    k = _normal(gen, (steps, N, H_qk, d_k), dtype)
    v = _normal(gen, (steps, N, H_v, d_v), dtype)
    la, b = _gates(gen, steps * N, H_v, "softplus01")
    g = _normal(gen, (steps, N, H_v, d_v), dtype) if epilogue else None
    w = (torch.randn((d_v,), generator=gen, dtype=torch.float32, device=gen.device) * 0.02
         if epilogue else None)
    return DecodeInputs(state, q, k, v, la.view(steps, N, H_v), b.view(steps, N, H_v),
                        g, w, meta={"seed": int(seed)})
