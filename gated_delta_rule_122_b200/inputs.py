"""Seeded synthetic inputs for the KDA workloads.

This module only draws random tensors; it holds none of the recurrence's
arithmetic, and both the CUDA path and the oracle consume the bytes it returns.

Workloads (name: shape; dtypes of q,k,v / alpha,beta; initial state):
  tiny     B=1 H=1   T=64    d=16   fp32 / fp32   zero
  small    B=1 H=4   T=2048  d=64   bf16 / fp32   N(0, 0.1)
  prefill  B=2 H=64  T=8192  d=128  bf16 / bf16   zero
  decode   N=256 H=64 (one token)   d=128  bf16 / bf16   N(0, 0.1)
  long     B=1 H=64  T=65536 d=128  bf16 / bf16   N(0, 0.1)

Distributions: q, k ~ N(0,1) then L2-normalised per token (in fp32, then cast);
v ~ N(0,1); beta = sigmoid(N(0,1)); alpha = exp(-softplus(x)) per key channel
and token, with x ~ N(0,1) (tiny, small, decode), 0.1*softplus(N(0,1)) in the
exponent (prefill), and for ``long`` a per-(head, key channel) Bernoulli(0.3)
mask choosing strong-forget channels exp(-softplus(N(2,1))) over near-one
channels exp(-0.1*softplus(N(0,1))).  Initial states are N(0, 0.1), i.e. std 0.1.
The seed is 1000 + the workload's index; draw order is q, k, v, beta, alpha,
[channel mask], initial state.  Streams are reproducible per (seed, device).
"""
from __future__ import annotations

import dataclasses

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "make_decode_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    qkv_dtype: torch.dtype
    gate_dtype: torch.dtype
    init_state: bool
    alpha_kind: str      # "unit_softplus", "near_one", "mixed"
    decode: bool = False

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def scaled(self, **over) -> "Workload":
        """Same distributions with some sizes overridden (e.g. a shorter T)."""
        return dataclasses.replace(self, **over)


WORKLOADS = {
    "tiny": Workload(0, "tiny", 1, 64, 1, 16, 16, torch.float32, torch.float32, False, "unit_softplus"),
    "small": Workload(1, "small", 1, 2048, 4, 64, 64, torch.bfloat16, torch.float32, True, "unit_softplus"),
    "prefill": Workload(2, "prefill", 2, 8192, 64, 128, 128, torch.bfloat16, torch.bfloat16, False, "near_one"),
    "decode": Workload(3, "decode", 256, 1, 64, 128, 128, torch.bfloat16, torch.bfloat16, True, "unit_softplus", True),
    "long": Workload(4, "long", 1, 65536, 64, 128, 128, torch.bfloat16, torch.bfloat16, True, "mixed"),
}


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, Workload):
        return name_or_index
    if isinstance(name_or_index, int):
        for w in WORKLOADS.values():
            if w.index == name_or_index:
                return w
        raise KeyError(name_or_index)
    return WORKLOADS[name_or_index]


def _unit_rows(g, shape, device):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x / x.norm(dim=-1, keepdim=True)


def _alpha(g, w: Workload, shape, device):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if w.alpha_kind == "unit_softplus":
        return torch.exp(-torch.nn.functional.softplus(x))
    if w.alpha_kind == "near_one":
        return torch.exp(-0.1 * torch.nn.functional.softplus(x))
    if w.alpha_kind == "mixed":
        near = torch.exp(-0.1 * torch.nn.functional.softplus(x))
        strong = torch.exp(-torch.nn.functional.softplus(
            torch.randn(shape, generator=g, device=device, dtype=torch.float32) + 2.0))
        # one Bernoulli(0.3) draw per (head, key channel), fixed over b and t
        H, dk = shape[-2], shape[-1]
        mask = torch.rand((H, dk), generator=g, device=device) < 0.3
        return torch.where(mask, strong, near)
    raise ValueError(w.alpha_kind)


def make_inputs(w, device="cpu", seed=None) -> dict:
    """Prefill inputs: q,k,alpha [B,T,H,dk], v [B,T,H,dv], beta [B,T,H], s0 [B,H,dk,dv] or None."""
    w = workload(w)
    assert not w.decode, "use make_decode_inputs for the decode workload"
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    q = _unit_rows(g, (B, T, H, dk), device).to(w.qkv_dtype)
    k = _unit_rows(g, (B, T, H, dk), device).to(w.qkv_dtype)
    v = torch.randn((B, T, H, dv), generator=g, device=device).to(w.qkv_dtype)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, device=device)).to(w.gate_dtype)
    alpha = _alpha(g, w, (B, T, H, dk), device).to(w.gate_dtype)
    s0 = None
    if w.init_state:
        s0 = 0.1 * torch.randn((B, H, dk, dv), generator=g, device=device, dtype=torch.float32)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, s0=s0, scale=dk ** -0.5, workload=w)


def make_decode_inputs(w="decode", device="cpu", seed=None) -> dict:
    """Decode inputs: q,k,alpha [N,H,dk], v [N,H,dv], beta [N,H], state [N,H,dk,dv] (fp32)."""
    w = workload(w)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    N, H, dk, dv = w.B, w.H, w.dk, w.dv
    q = _unit_rows(g, (N, H, dk), device).to(w.qkv_dtype)
    k = _unit_rows(g, (N, H, dk), device).to(w.qkv_dtype)
    v = torch.randn((N, H, dv), generator=g, device=device).to(w.qkv_dtype)
    beta = torch.sigmoid(torch.randn((N, H), generator=g, device=device)).to(w.gate_dtype)
    alpha = _alpha(g, w, (N, H, dk), device).to(w.gate_dtype)
    state = 0.1 * torch.randn((N, H, dk, dv), generator=g, device=device, dtype=torch.float32)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, state=state, scale=dk ** -0.5, workload=w)
