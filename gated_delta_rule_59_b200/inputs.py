"""Seeded synthetic inputs shared by the tests, the bench and the oracle legs.

This module holds only random-number recipes and shapes: none of the
recurrence's arithmetic.  Everything is drawn on the CPU with
``torch.Generator().manual_seed(seed)`` in float32, q and k are L2-normalised
per head (the "DeltaNet Attention" page normalises queries and keys before the
rule; the "DeltaNet" block diagram puts an L2 norm in front of it), and then
cast to the working dtype.  The oracle receives exactly the cast values,
upcast to float64.

Workloads (shapes from the "linear_attention" page: q, k [batch, seq, heads,
key_dim]; v [batch, seq, heads, value_dim]; decays and betas [batch, seq,
heads] float32):

  0  plain DeltaNet, fp32: B=1 T=64 H=2 d=16, g = 0, zero initial state
  1  DeltaNet layer: B=4 T=2048 H=16 d=64, bf16, g = 0, zero initial state
  2  gated prefill (Qwen3-Next-like): B=2 T=8192 Hqk=16 -> Hv=32 d=128, bf16,
     g = log(sigmoid(x)), x ~ N(3,1); beta = sigmoid(N(0,1)); state ~ N(0, 0.02^2)
  3  gated decode: B=256 H=32 d=128, bf16, g as in 2, beta = 2 sigmoid(N(0,1)),
     cached fp32 state ~ N(0, 0.02^2), 64 consecutive steps with fresh inputs
  4  varlen gated prefill: 8 lengths uniform in [512, 16384] + one of 65536,
     packed with cu_seqlens (B=1), H=16 d=128, bf16, g/beta/state as in 2

Per-key-channel gates (``channel_gates=True``, the "linear_attention" page's
ChannelGates [batch, seq, heads, key_dim]) draw g per channel from the same
distribution as the scalar gate, in place of it.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

SEED_BASE = 1000


@dataclasses.dataclass
class Prefill:
    q: torch.Tensor  # [B, T, Hqk, dk]
    k: torch.Tensor  # [B, T, Hqk, dk]
    v: torch.Tensor  # [B, T, Hv, dv]
    g: Optional[torch.Tensor]  # [B, T, Hv] (or [B, T, Hv, dk]: per key channel) float32 or None
    beta: torch.Tensor  # [B, T, Hv] float32
    state_in: Optional[torch.Tensor]  # [N, Hv, dk, dv] float32 or None
    cu_seqlens: Optional[torch.Tensor]  # int32 [N+1] or None
    name: str = ""

    @property
    def n_tokens(self) -> int:
        return int(self.q.shape[0] * self.q.shape[1])

    def to(self, device):
        f = lambda t: None if t is None else t.to(device, non_blocking=True)
        return Prefill(f(self.q), f(self.k), f(self.v), f(self.g), f(self.beta),
                       f(self.state_in), f(self.cu_seqlens), self.name)


def _gen(seed: int) -> torch.Generator:
    gen = torch.Generator()
    gen.manual_seed(seed)
    return gen


def _l2(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _qk(gen, shape, dtype):
    return _l2(torch.randn(shape, generator=gen)).to(dtype)


def _log_sigmoid_gate(gen, shape):
    # g = log(sigmoid(x)), x ~ N(3, 1): float32 and non-positive.
    x = torch.randn(shape, generator=gen) + 3.0
    return torch.nn.functional.logsigmoid(x).float()


def prefill(B, T, Hqk, Hv, dk, dv, dtype=torch.bfloat16, gated=True, beta_max=1.0,
            state_std=0.0, seed=0, cu_seqlens=None, name="", channel_gates=False) -> Prefill:
    """Generic seeded prefill problem (the shapes and distributions above)."""
    gen = _gen(seed)
    q = _qk(gen, (B, T, Hqk, dk), dtype)
    k = _qk(gen, (B, T, Hqk, dk), dtype)
    v = torch.randn((B, T, Hv, dv), generator=gen).to(dtype)
    beta = (beta_max * torch.sigmoid(torch.randn((B, T, Hv), generator=gen))).float()
    g = _log_sigmoid_gate(gen, (B, T, Hv) + ((dk,) if channel_gates else ())) if gated else None
    N = B if cu_seqlens is None else len(cu_seqlens) - 1
    state = None
    if state_std > 0:
        state = (state_std * torch.randn((N, Hv, dk, dv), generator=gen)).float()
    cu = None if cu_seqlens is None else torch.tensor(cu_seqlens, dtype=torch.int32)
    return Prefill(q, k, v, g, beta, state, cu, name)


def varlen_lengths(seed: int, n_short: int = 8, lo: int = 512, hi: int = 16384,
                   long_len: int = 65536):
    gen = _gen(seed + 7)
    lens = torch.randint(lo, hi + 1, (n_short,), generator=gen).tolist()
    return lens + ([long_len] if long_len else [])


def cu_from_lengths(lens):
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    return cu


def config(idx: int, seed: Optional[int] = None) -> Prefill:
    """Prefill workloads 0, 1, 2 and 4 (3 is the decode workload: ``decode_config``)."""
    s = SEED_BASE + idx if seed is None else seed
    if idx == 0:
        return prefill(1, 64, 2, 2, 16, 16, torch.float32, gated=False, seed=s,
                       name="deltanet_fp32_B1_T64_H2_d16")
    if idx == 1:
        return prefill(4, 2048, 16, 16, 64, 64, torch.bfloat16, gated=False, seed=s,
                       name="deltanet_bf16_B4_T2048_H16_d64")
    if idx == 2:
        return prefill(2, 8192, 16, 32, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=s, name="gated_prefill_bf16_B2_T8192_Hqk16_Hv32_d128")
    if idx == 4:
        lens = varlen_lengths(s)
        cu = cu_from_lengths(lens)
        return prefill(1, cu[-1], 16, 16, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=s, cu_seqlens=cu, name="varlen_gated_prefill_bf16_H16_d128")
    raise ValueError(f"no prefill workload {idx}")


@dataclasses.dataclass
class DecodeStep:
    q: torch.Tensor  # [B, Hqk, dk]
    k: torch.Tensor  # [B, Hqk, dk]
    v: torch.Tensor  # [B, Hv, dv]
    g: Optional[torch.Tensor]  # [B, Hv] (or [B, Hv, dk]: per key channel)
    beta: torch.Tensor  # [B, Hv]

    def to(self, device):
        f = lambda t: None if t is None else t.to(device, non_blocking=True)
        return DecodeStep(f(self.q), f(self.k), f(self.v), f(self.g), f(self.beta))


def decode_state(B, Hv, dk, dv, std=0.02, seed=0) -> torch.Tensor:
    gen = _gen(seed)
    return (std * torch.randn((B, Hv, dk, dv), generator=gen)).float()


def decode_steps(B, Hqk, Hv, dk, dv, n_steps, dtype=torch.bfloat16, gated=True,
                 beta_max=2.0, seed=0, channel_gates=False):
    """``n_steps`` fresh seeded decode inputs (one token per sequence each)."""
    gen = _gen(seed + 1)
    out = []
    for _ in range(n_steps):
        q = _qk(gen, (B, Hqk, dk), dtype)
        k = _qk(gen, (B, Hqk, dk), dtype)
        v = torch.randn((B, Hv, dv), generator=gen).to(dtype)
        beta = (beta_max * torch.sigmoid(torch.randn((B, Hv), generator=gen))).float()
        g = _log_sigmoid_gate(gen, (B, Hv) + ((dk,) if channel_gates else ())) if gated else None
        out.append(DecodeStep(q, k, v, g, beta))
    return out


def decode_config(n_steps: int = 64, B: int = 256, seed: Optional[int] = None):
    """Workload 3: returns (state [B, 32, 128, 128] fp32, list of DecodeStep)."""
    s = SEED_BASE + 3 if seed is None else seed
    state = decode_state(B, 32, 128, 128, 0.02, seed=s)
    steps = decode_steps(B, 32, 32, 128, 128, n_steps, torch.bfloat16, True, 2.0, seed=s)
    return state, steps
