"""Seeded synthetic inputs for the gated delta rule forward pass and decode step.

This module holds random draws only: no step of the recurrence or of the
chunkwise algorithm lives here. Both the CUDA path (tests, bench) and the CPU
oracle (tests) take their inputs from it, so the two sides see the same bytes.

Workload shapes and distributions follow the synthetic configurations this
library is measured on:

* ``tiny_fp32``  B=1 H=2 T=256 d=64, fp32 inputs, zero initial state, seed 0
* ``b4h16t4096`` B=4 H=16 T=4096 d=128, bf16 q/k/v, zero initial state, seed 1
* ``long64k``    B=1 H=16 T=65536 d=128, bf16, slow decay, random state, seed 2
* ``varlen64``   64 packed sequences, lengths log-uniform in [128, 2048], H=32
* ``decode``     N=256 H=32 d=128 fp32 state, 64 consecutive single-token steps
* ``b4h16t4096_beta2`` the b4h16t4096 shape with beta = 2 sigmoid(N(0, 1)) in
  (0, 2): the negative-eigenvalue range of I - beta k k^T, seed 5
* ``kda_b4h16t4096`` the b4h16t4096 shape with the channel-wise gate (one
  log-decay per d_k channel, g [B,T,H,d_k]), seed 6
* ``kda_decode``  the decode shape with the channel-wise gate, seed 7
* ``b1h16t1024``  one sequence of the b4h16t4096 kind, 1024 tokens, seed 8: a
  small case of the same kernels for full profiler captures
* ``kda_b1h16t1024`` the same with the channel-wise gate, seed 9

Distributions (all drawn in fp32 with ``torch.Generator('cpu')``):
q, k ~ N(0, 1) then L2-normalised per (token, head) over d_k; v ~ N(0, 1);
beta = sigmoid(N(0, 1)); g = log(alpha) = -softplus(N(mu, 1)) with mu = -2
(mu = -4 for the long-context workload), drawn per token and head, or per
token, head and d_k channel for the channel-wise gate; random states
~ N(0, 0.02) (std). Draw order: lengths (varlen only), q, k, v, beta-logits,
g-normal, state.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "make_chunk_inputs", "make_decode_inputs",
           "varlen_lengths"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    chunk: int = 64
    dtype: torch.dtype = torch.bfloat16
    gate_mu: float = -2.0
    random_state: bool = False
    seed: int = 0
    num_seqs: int = 0          # >0: packed variable-length batch (B must be 1)
    len_range: tuple = field(default=(128, 2048))
    steps: int = 1             # decode workloads: consecutive steps
    beta_scale: float = 1.0    # beta = beta_scale * sigmoid(N(0, 1))
    gate: str = "scalar"       # "scalar": g [..., H]; "channel": g [..., H, d_k]


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, T=256, H=2, d_k=64, d_v=64,
                          dtype=torch.float32, seed=0),
    "b4h16t4096": Workload("b4h16t4096", B=4, T=4096, H=16, d_k=128, d_v=128, seed=1),
    "long64k": Workload("long64k", B=1, T=65536, H=16, d_k=128, d_v=128,
                        gate_mu=-4.0, random_state=True, seed=2),
    "varlen64": Workload("varlen64", B=1, T=0, H=32, d_k=128, d_v=128, seed=3,
                         num_seqs=64),
    "decode": Workload("decode", B=256, T=1, H=32, d_k=128, d_v=128,
                       random_state=True, seed=4, steps=64),
    "b4h16t4096_beta2": Workload("b4h16t4096_beta2", B=4, T=4096, H=16, d_k=128, d_v=128,
                                 seed=5, beta_scale=2.0),
    "kda_b4h16t4096": Workload("kda_b4h16t4096", B=4, T=4096, H=16, d_k=128, d_v=128,
                               seed=6, gate="channel"),
    "b1h16t1024": Workload("b1h16t1024", B=1, T=1024, H=16, d_k=128, d_v=128, seed=8),
    "kda_decode": Workload("kda_decode", B=256, T=1, H=32, d_k=128, d_v=128,
                           random_state=True, seed=7, steps=64, gate="channel"),
    "kda_b1h16t1024": Workload("kda_b1h16t1024", B=1, T=1024, H=16, d_k=128, d_v=128, seed=9,
                               gate="channel"),
}


def varlen_lengths(gen: torch.Generator, num_seqs: int, lo: int, hi: int) -> list[int]:
    """Lengths log-uniform in [lo, hi]: floor(exp(U(ln lo, ln hi))), clamped."""
    u = torch.rand(num_seqs, generator=gen, dtype=torch.float32)
    x = torch.exp(math.log(lo) + u.double() * (math.log(hi) - math.log(lo)))
    return [int(min(max(math.floor(float(v)), lo), hi)) for v in x]


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # L2-normalise the last dimension in fp32 (input preparation, as specified
    # by the workloads; the kernels never normalise).
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _gates(gen, shape, mu, beta_scale=1.0, g_shape=None):
    beta = beta_scale * torch.sigmoid(torch.randn(shape, generator=gen, dtype=torch.float32))
    g = -torch.nn.functional.softplus(
        torch.randn(shape if g_shape is None else g_shape, generator=gen,
                    dtype=torch.float32) + mu)
    return g.contiguous(), beta.contiguous()


def _g_shape(w, shape):
    return tuple(shape) + (w.d_k,) if w.gate == "channel" else None


def make_chunk_inputs(w: Workload | str, *, seed: int | None = None, T: int | None = None,
                      B: int | None = None, H: int | None = None,
                      lengths: list[int] | None = None, dtype: torch.dtype | None = None,
                      random_state: bool | None = None, gate_mu: float | None = None):
    """Draw one batch for the chunked forward pass (CPU tensors).

    Returns a dict with q, k ``[B,T,H,d_k]``, v ``[B,T,H,d_v]`` in the workload
    dtype, g and beta ``[B,T,H]`` fp32 (g ``[B,T,H,d_k]`` for the channel-wise
    gate), ``initial_state`` ``[N,H,d_k,d_v]`` fp32
    or None, ``cu_seqlens`` int32 ``[N+1]`` or None, and the workload fields.
    Keyword overrides shrink a workload for tests (same distributions).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    seed = w.seed if seed is None else seed
    H = w.H if H is None else H
    dtype = w.dtype if dtype is None else dtype
    random_state = w.random_state if random_state is None else random_state
    gate_mu = w.gate_mu if gate_mu is None else gate_mu
    gen = torch.Generator("cpu").manual_seed(seed)
    cu = None
    if lengths is None and w.num_seqs > 0:
        lengths = varlen_lengths(gen, w.num_seqs, *w.len_range)
    if lengths is not None:
        Bn, Tn = 1, int(sum(lengths))
        cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0).tolist()),
                          dtype=torch.int32)
        N = len(lengths)
    else:
        Bn = w.B if B is None else B
        Tn = w.T if T is None else T
        N = Bn
    q = _unit_rows(torch.randn(Bn, Tn, H, w.d_k, generator=gen, dtype=torch.float32))
    k = _unit_rows(torch.randn(Bn, Tn, H, w.d_k, generator=gen, dtype=torch.float32))
    v = torch.randn(Bn, Tn, H, w.d_v, generator=gen, dtype=torch.float32)
    g, beta = _gates(gen, (Bn, Tn, H), gate_mu, w.beta_scale, _g_shape(w, (Bn, Tn, H)))
    s0 = None
    if random_state:
        s0 = 0.02 * torch.randn(N, H, w.d_k, w.d_v, generator=gen, dtype=torch.float32)
    return dict(q=q.to(dtype).contiguous(), k=k.to(dtype).contiguous(),
                v=v.to(dtype).contiguous(), g=g, beta=beta, initial_state=s0,
                cu_seqlens=cu, chunk=w.chunk, B=Bn, T=Tn, H=H, d_k=w.d_k, d_v=w.d_v,
                num_seqs=N, dtype=dtype, gate=w.gate)


def make_decode_inputs(w: Workload | str = "decode", *, seed: int | None = None,
                       N: int | None = None, H: int | None = None, steps: int | None = None,
                       dtype: torch.dtype | None = None):
    """Draw the initial state and ``steps`` single-token inputs (CPU tensors).

    Returns dict(state ``[N,H,d_k,d_v]`` fp32, q/k ``[steps,N,H,d_k]``,
    v ``[steps,N,H,d_v]``, g/beta ``[steps,N,H]`` fp32, g ``[steps,N,H,d_k]``
    for the channel-wise gate). The state is drawn
    first, then each step's q, k, v, beta-logits, g-normal in step order.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    seed = w.seed if seed is None else seed
    N = w.B if N is None else N
    H = w.H if H is None else H
    steps = w.steps if steps is None else steps
    dtype = w.dtype if dtype is None else dtype
    gen = torch.Generator("cpu").manual_seed(seed)
    state = 0.02 * torch.randn(N, H, w.d_k, w.d_v, generator=gen, dtype=torch.float32)
    qs, ks, vs, gs, bs = [], [], [], [], []
    for _ in range(steps):
        qs.append(_unit_rows(torch.randn(N, H, w.d_k, generator=gen, dtype=torch.float32)))
        ks.append(_unit_rows(torch.randn(N, H, w.d_k, generator=gen, dtype=torch.float32)))
        vs.append(torch.randn(N, H, w.d_v, generator=gen, dtype=torch.float32))
        g, b = _gates(gen, (N, H), w.gate_mu, 1.0, _g_shape(w, (N, H)))
        gs.append(g)
        bs.append(b)
    return dict(state=state.contiguous(),
                q=torch.stack(qs).to(dtype).contiguous(),
                k=torch.stack(ks).to(dtype).contiguous(),
                v=torch.stack(vs).to(dtype).contiguous(),
                g=torch.stack(gs).contiguous(), beta=torch.stack(bs).contiguous(),
                N=N, H=H, d_k=w.d_k, d_v=w.d_v, steps=steps, dtype=dtype, gate=w.gate)
