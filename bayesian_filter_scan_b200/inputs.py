"""Seeded synthetic inputs for the Kalman linear-attention forward pass.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It draws random numbers and shapes them into the filter's
inputs; it holds none of the filter's arithmetic (no predict, update, gate or
readout step appears here).

Workloads follow the shapes the Kalman Linear Attention and Kalman Delta
Network pages speak of: layers of 750M-1.3B-class models (Kalman Delta
Networks abstract), the 2048-token associative-recall length (KLA technical
summary, experiments), and 128k-token contexts (Gated KalmaNet abstract).
There is no dataset; every tensor is drawn from a ``torch.Generator('cpu')``.

Layout (row-major, tokens flattened over the batch):
  q, k            [B*T, H, dk]   bf16 (fp32 for the fp32 workload)
  v               [B*T, H, dv]
  a, qn           [B*T, H, dk]   fp32 (isotropic mode: [B*T, H])
  beta            [B*T, H]       fp32
  lambda0         [N, H, dk]     fp32 (isotropic: [N, H]); N = B or #sequences
  eta0            [N, H, dk, dv] fp32
  cu_seqlens      int32 [N+1] offsets into the flattened token axis, or None
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: str = "bf16"          # dtype of q, k, v, out: "bf16" or "fp32"
    mode: str = "diag"           # "diag" (precision per key) or "iso" (per head)
    a_mu: float = 2.0            # a = sigmoid(N(a_mu, 1)) (diagonal workloads)
    qn_mu: float = -2.0          # qn = softplus(N(qn_mu, 1))
    varlen: bool = False         # packed variable-length sequences
    len_lo: int = 512            # varlen: sequence lengths ~ U{len_lo..len_hi}
    len_hi: int = 8192
    final_state: bool = False    # the workload asks for final_lambda/final_eta
    seed: int = 0
    iso_sigmoid: bool = False    # isotropic mode: a = sigmoid(N(a_mu, 1)), qn = softplus(N(qn_mu, 1))
                                 # per (t,h) instead of the near-unit stress gates

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: tiny fp32, small layer, 1.3B-class layer, 128k context,
# isotropic stress with packed sequences.
WORKLOADS = {
    0: Workload("tiny-fp32", B=1, H=2, T=256, dk=16, dv=16, dtype="fp32",
                a_mu=2.0, qn_mu=-2.0, seed=0),
    1: Workload("small-layer", B=4, H=8, T=2048, dk=64, dv=64,
                a_mu=2.0, qn_mu=-2.0, seed=1),
    2: Workload("1.3B-layer", B=8, H=16, T=4096, dk=128, dv=128,
                a_mu=3.0, qn_mu=-3.0, seed=2),
    3: Workload("long-context-128k", B=1, H=16, T=131072, dk=128, dv=128,
                a_mu=3.0, qn_mu=-3.0, final_state=True, seed=3),
    4: Workload("iso-varlen-stress", B=2, H=32, T=16384, dk=64, dv=128,
                mode="iso", varlen=True, final_state=True, seed=4),
}


def varlen_offsets(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """Packed sequence offsets: each batch row of T tokens is filled with
    lengths drawn from U{len_lo..len_hi}; the last sequence of a row is cut
    at the row's end. Returns int32 offsets into the flattened token axis."""
    offs = [0]
    for b in range(w.B):
        filled = 0
        while filled < w.T:
            n = int(torch.randint(w.len_lo, w.len_hi + 1, (1,), generator=gen).item())
            n = min(n, w.T - filled)
            filled += n
            offs.append(b * w.T + filled)
    return torch.tensor(offs, dtype=torch.int32)


def make_inputs(w: Workload, seed: Optional[int] = None) -> dict:
    """Draw the inputs of workload ``w`` on the CPU. Floating-point values are
    drawn in fp32 and cast once to the input dtype, so the copy sent to the GPU
    and the copy the oracle upcasts hold identical values."""
    gen = torch.Generator("cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    N_tok, H, dk, dv = w.tokens, w.H, w.dk, w.dv
    io = torch.float32 if w.dtype == "fp32" else torch.bfloat16

    def unit_rows(x):
        return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)

    q = unit_rows(torch.randn(N_tok, H, dk, generator=gen)).to(io)
    k = unit_rows(torch.randn(N_tok, H, dk, generator=gen)).to(io)
    v = torch.randn(N_tok, H, dv, generator=gen).to(io)
    if w.mode == "iso" and w.iso_sigmoid:
        a = torch.sigmoid(w.a_mu + torch.randn(N_tok, H, generator=gen))
        qn = torch.nn.functional.softplus(w.qn_mu + torch.randn(N_tok, H, generator=gen))
        beta = torch.sigmoid(torch.randn(N_tok, H, generator=gen))
    elif w.mode == "iso":
        a = 1.0 - 1e-4 * torch.rand(N_tok, H, generator=gen)
        qn = torch.full((N_tok, H), 1e-4)
        lo, hi = math.log(0.5), math.log(8.0)
        beta = torch.exp(lo + (hi - lo) * torch.rand(N_tok, H, generator=gen))
    else:
        a = torch.sigmoid(w.a_mu + torch.randn(N_tok, H, dk, generator=gen))
        qn = torch.nn.functional.softplus(w.qn_mu + torch.randn(N_tok, H, dk, generator=gen))
        beta = torch.sigmoid(torch.randn(N_tok, H, generator=gen))
    cu = varlen_offsets(w, gen) if w.varlen else None
    N = (cu.numel() - 1) if cu is not None else w.B
    lam_shape = (N, H) if w.mode == "iso" else (N, H, dk)
    return dict(
        q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
        a=a.float().contiguous(), qn=qn.float().contiguous(), beta=beta.float().contiguous(),
        lambda0=torch.ones(lam_shape), eta0=torch.zeros(N, H, dk, dv),
        cu_seqlens=cu,
    )


def random_state(w: Workload, N: int, seed: int) -> tuple:
    """A non-trivial starting belief (lambda0 > 0, eta0 arbitrary) for tests
    of the state hand-off."""
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    lam_shape = (N, w.H) if w.mode == "iso" else (N, w.H, w.dk)
    lam0 = 0.5 + 2.0 * torch.rand(lam_shape, generator=gen)
    eta0 = torch.randn(N, w.H, w.dk, w.dv, generator=gen)
    return lam0.contiguous(), eta0.contiguous()
