"""Seeded synthetic inputs for the KDA entry points.

This module serves both the CUDA path and the fp64 oracle.  It holds none of
the method's arithmetic: it only draws random tensors and applies the input
transforms that sit upstream of the token mixer in the model (L2-normalised
q/k, q scaled by 1/sqrt(dk), beta = sigmoid(.), g = -softplus(.)/c).  Those
transforms are part of the workload description, not of the recurrence.

All draws use ``torch.Generator('cpu').manual_seed(seed)``; tensors are drawn
in fp32 in a fixed order (q, k, v, g-noise, beta-noise, then extras), then
transformed, then cast (q, k, v to the compute dtype; g, beta, states stay
fp32).

Named workloads (sizes as the Kimi Linear pages' decode/prefill discussion
motivates; the pages print no shapes of their own):
  prefill_t256_h1_d64_f32     B=1 H=1  T=256    d=64  fp32, seed 0
  prefill_t8192_h32_d128      B=1 H=32 T=8192   d=128 bf16, seed 1
  prefill_t65536_h32_d128     B=1 H=32 T=65536  d=128 bf16, seed 2
                              (per-channel offset gate: long- and
                              short-memory channels)
  varlen8_h32_d128_resume     8 packed sequences, lengths U[1024, 32768],
                              H=32 d=128 bf16, initial states 0.02*N(0,1),
                              seed 3
  decode_n256_h32_d128        256 sequences x H=32, d=128 bf16 tokens, fp32
                              state 0.02*N(0,1), seed 4; token inputs of step
                              t come from seed (4, t)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass
class PrefillInputs:
    q: torch.Tensor            # [B,T,H,dk]
    k: torch.Tensor            # [B,T,H,dk]
    v: torch.Tensor            # [B,T,H,dv]
    g: torch.Tensor            # [B,T,H,dk] fp32, log alpha
    beta: torch.Tensor         # [B,T,H] fp32
    initial_state: torch.Tensor | None   # [N,H,dk,dv] fp32 or None
    cu_seqlens: torch.Tensor | None      # [N+1] int32 or None
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return self.q.shape[0] if self.cu_seqlens is None else self.cu_seqlens.numel() - 1

    def to(self, device) -> "PrefillInputs":
        mv = lambda t: None if t is None else t.to(device)
        return PrefillInputs(mv(self.q), mv(self.k), mv(self.v), mv(self.g),
                             mv(self.beta), mv(self.initial_state),
                             mv(self.cu_seqlens), dict(self.meta))


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def draw_tokens(gen: torch.Generator, lead: tuple, dk: int, dv: int,
                dtype: torch.dtype, gate: str = "softplus8", H: int | None = None):
    """Draw q, k, v, g, beta for token positions of shape ``lead`` (ending in H).

    gate = "softplus8":  g = -softplus(z)/8, z ~ N(0,1)
    gate = "offset16":   g = -softplus(z + 2 + off[h,c])/16 with
                         off ~ U(-3,3) per (head, channel), drawn after beta.
    """
    q = torch.randn(*lead, dk, generator=gen)
    k = torch.randn(*lead, dk, generator=gen)
    v = torch.randn(*lead, dv, generator=gen)
    gz = torch.randn(*lead, dk, generator=gen)
    bz = torch.randn(*lead, generator=gen)
    q = _l2norm(q) * (1.0 / math.sqrt(dk))
    k = _l2norm(k)
    if gate == "softplus8":
        g = -F.softplus(gz) / 8.0
    elif gate == "offset16":
        Hh = lead[-1] if H is None else H
        off = torch.rand(Hh, dk, generator=gen) * 6.0 - 3.0
        g = -F.softplus(gz + 2.0 + off) / 16.0
    elif gate == "zero":
        g = torch.zeros_like(gz)
    else:
        raise ValueError(gate)
    beta = torch.sigmoid(bz)
    return (q.to(dtype), k.to(dtype), v.to(dtype), g.float().contiguous(),
            beta.float().contiguous())


def prefill(B: int, T: int, H: int, dk: int = 128, dv: int = 128,
            dtype: torch.dtype = torch.bfloat16, seed: int = 0,
            gate: str = "softplus8", initial_state_std: float | None = None,
            seq_lens: list[int] | None = None) -> PrefillInputs:
    """Dense [B,T,H,*] inputs, or (seq_lens given) one packed varlen batch."""
    gen = torch.Generator("cpu").manual_seed(seed)
    cu = None
    if seq_lens is not None:
        B, T = 1, int(sum(seq_lens))
        cu = torch.zeros(len(seq_lens) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(seq_lens, dtype=torch.int64), 0).to(torch.int32)
    q, k, v, g, beta = draw_tokens(gen, (B, T, H), dk, dv, dtype, gate)
    N = B if cu is None else cu.numel() - 1
    s0 = None
    if initial_state_std is not None:
        s0 = (torch.randn(N, H, dk, dv, generator=gen) * initial_state_std).float()
    return PrefillInputs(q, k, v, g, beta, s0, cu,
                         dict(B=B, T=T, H=H, dk=dk, dv=dv, seed=seed, gate=gate))


def varlen_lengths(seed: int = 3, n: int = 8, lo: int = 1024, hi: int = 32768) -> list[int]:
    gen = torch.Generator("cpu").manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]


def named_prefill(name: str) -> PrefillInputs:
    if name == "prefill_t256_h1_d64_f32":
        return prefill(1, 256, 1, 64, 64, torch.float32, seed=0)
    if name == "prefill_t8192_h32_d128":
        return prefill(1, 8192, 32, 128, 128, torch.bfloat16, seed=1)
    if name == "prefill_t65536_h32_d128":
        return prefill(1, 65536, 32, 128, 128, torch.bfloat16, seed=2, gate="offset16")
    if name == "varlen8_h32_d128_resume":
        lens = varlen_lengths(3)
        # lengths are drawn first from seed 3; token draws continue from seed 3
        # in a generator of their own (documented recipe)
        return prefill(1, 0, 32, 128, 128, torch.bfloat16, seed=3,
                       initial_state_std=0.02, seq_lens=lens)
    raise KeyError(name)


DECODE_N, DECODE_H, DECODE_D, DECODE_SEED = 256, 32, 128, 4


def decode_initial_state(N: int = DECODE_N, H: int = DECODE_H, dk: int = DECODE_D,
                         dv: int = DECODE_D, seed: int = DECODE_SEED,
                         std: float = 0.02) -> torch.Tensor:
    gen = torch.Generator("cpu").manual_seed(seed)
    return (torch.randn(N, H, dk, dv, generator=gen) * std).float()


def decode_tokens(step: int, N: int = DECODE_N, H: int = DECODE_H, dk: int = DECODE_D,
                  dv: int = DECODE_D, dtype: torch.dtype = torch.bfloat16,
                  seed: int = DECODE_SEED, gate: str = "softplus8"):
    """Token inputs of decode step ``step``: q,k [N,H,dk], v [N,H,dv], g, beta."""
    gen = torch.Generator("cpu").manual_seed(seed * 1_000_003 + 7919 * (step + 1))
    return draw_tokens(gen, (N, H), dk, dv, dtype, gate)
