"""Seeded synthetic inputs for KDA, shared by the tests, the bench and the smoke check.

This module holds none of the method's arithmetic: it only draws random
tensors with the distributions of the workloads and prepares them the way a
KDA layer hands them to the operator (blog.gzher.com "Kimi K3论文：Kimi
Linear", section 3, neural parameterisation: q and k are L2-normalised per
head, beta is a sigmoid, alpha lies in [0, 1] per key channel so the operator
takes log_alpha <= 0).

Recipe (every draw from one ``torch.Generator`` seeded with ``seed``, in the
order listed, on ``device``):
  q, k       ~ N(0, 1), L2-normalised over the key dimension, cast to ``dtype``
  v          ~ N(0, 1), cast to ``dtype``
  log_alpha  = -U(lo, hi), fp32, independent per (token, head, key channel); with
               gate="head" one per (token, head), with gate="channel_bf16" the
               same draw cast to bf16, with gate="none" no draw (None)
  beta       = sigmoid(N(0, 1)), fp32, one per (token, head)
  S0         ~ N(0, s0_std^2) fp32 per (sequence, head, dk, dv); zeros if s0_std == 0
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

DK = 128
DV = 128


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: torch.Tensor | None  # in the layout of `gate` (GATES)
    beta: torch.Tensor
    S0: torch.Tensor | None
    cu_seqlens: torch.Tensor | None  # int32 [n_seqs + 1] on the inputs' device, or None
    gate: str = "channel"

    @property
    def n_seqs(self) -> int:
        return self.q.shape[0] if self.cu_seqlens is None else self.cu_seqlens.numel() - 1


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit_normal_rows(shape, gen, device, dtype) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    return x.to(dtype)


# Forget-gate layouts (the library's kda_gate): per key channel in fp32 or bf16, one per
# (token, head) in fp32, or none. Values are drawn as -U(lo, hi) in fp32.
GATES = ("channel", "channel_bf16", "head", "none")


def _draw_gate(gate: str, lead, H: int, dk: int, la_range, gen, device):
    lo, hi = la_range
    if gate == "none":
        return None
    shape = lead + ((H,) if gate == "head" else (H, dk))
    la = -(lo + (hi - lo) * torch.rand(shape, generator=gen, device=device, dtype=torch.float32))
    return la.to(torch.bfloat16) if gate == "channel_bf16" else la


def varlen_lengths(n_seqs: int, lo: int, hi: int, seed: int) -> list[int]:
    """Sequence lengths drawn uniformly from the integers [lo, hi] (CPU generator)."""
    g = _gen(seed, "cpu")
    return torch.randint(lo, hi + 1, (n_seqs,), generator=g).tolist()


def cu_from_lengths(lengths, device="cpu") -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def prefill_inputs(*, T: int, H: int, B: int = 1, cu_seqlens=None, dtype=torch.bfloat16,
                   la_range=(0.001, 0.1), s0_std: float = 0.0, seed: int = 0,
                   device="cpu", dk: int = DK, dv: int = DV, gate: str = "channel") -> PrefillInputs:
    """Inputs for one ``kda_chunk_fwd`` call.

    Without ``cu_seqlens`` the tensors are ``[B, T, H, .]``; with it (a list or
    tensor of ``n_seqs + 1`` offsets ending at ``T``) they are packed
    ``[T, H, .]`` and ``B`` must be 1. ``gate`` picks the layout of
    ``log_alpha`` (one of GATES).
    """
    gen = _gen(seed, device)
    if cu_seqlens is None:
        lead = (B, T)
        n_seqs = B
        cu = None
    else:
        assert B == 1
        cu = torch.as_tensor(cu_seqlens, dtype=torch.int32).to(device)
        assert int(cu[-1]) == T
        lead = (T,)
        n_seqs = cu.numel() - 1
    q = _unit_normal_rows(lead + (H, dk), gen, device, dtype)
    k = _unit_normal_rows(lead + (H, dk), gen, device, dtype)
    v = torch.randn(lead + (H, dv), generator=gen, device=device, dtype=torch.float32).to(dtype)
    la = _draw_gate(gate, lead, H, dk, la_range, gen, device)
    beta = torch.sigmoid(torch.randn(lead + (H,), generator=gen, device=device, dtype=torch.float32))
    S0 = None
    if s0_std > 0:
        S0 = s0_std * torch.randn((n_seqs, H, dk, dv), generator=gen, device=device, dtype=torch.float32)
    return PrefillInputs(q, k, v, la, beta, S0, cu, gate)


@dataclass
class DecodeInputs:
    q: torch.Tensor          # [steps, N, H, dk]
    k: torch.Tensor          # [steps, N, H, dk]
    v: torch.Tensor          # [steps, N, H, dv]
    log_alpha: torch.Tensor | None  # [steps, N, H, dk] fp32 (layout of `gate`)
    beta: torch.Tensor       # [steps, N, H] fp32
    S: torch.Tensor          # [N, H, dk, dv] fp32 initial state
    gate: str = "channel"


def decode_inputs(*, steps: int, N: int, H: int, dtype=torch.bfloat16, la_range=(0.001, 0.1),
                  s0_std: float = 0.1, seed: int = 0, device="cpu", dk: int = DK,
                  dv: int = DV, gate: str = "channel") -> DecodeInputs:
    """Per-step token inputs for ``steps`` consecutive ``kda_decode_step`` calls."""
    gen = _gen(seed, device)
    lead = (steps, N)
    q = _unit_normal_rows(lead + (H, dk), gen, device, dtype)
    k = _unit_normal_rows(lead + (H, dk), gen, device, dtype)
    v = torch.randn(lead + (H, dv), generator=gen, device=device, dtype=torch.float32).to(dtype)
    la = _draw_gate(gate, lead, H, dk, la_range, gen, device)
    beta = torch.sigmoid(torch.randn(lead + (H,), generator=gen, device=device, dtype=torch.float32))
    S = s0_std * torch.randn((N, H, dk, dv), generator=gen, device=device, dtype=torch.float32)
    return DecodeInputs(q, k, v, la, beta, S, gate)
