"""Seeded synthetic inputs for the ZeRO step (shared by tests, bench and smoke).

This module only draws random numbers and lays them out in the padded logical
order (unit u occupies [U_u, U_u + P_u), its first len_u entries real, the
rest zero).  It holds none of the method's arithmetic and imports neither the
CUDA library nor the oracle, so both sides can be fed the same bytes.

Recipe (per config; seed = 1000*config + 10*rank + step):
  gradients  fp32 N(0, sigma) drawn per rank, optionally with a Bernoulli
             fraction of entries multiplied by `outlier_scale`, then rounded
             to bf16 (torch's round-to-nearest-even); padding zero.
  master     fp32 N(0, 0.02) in logical order, padding zero (seed from
             `master_seed`); m = v = 0.
"""
from typing import List, Optional

import torch


def seed_for(config: int, rank: int, step: int) -> int:
    return 1000 * config + 10 * rank + step


def master_seed(config: int) -> int:
    return 1000 * config + 999


def _fill_padded(dst: torch.Tensor, src: torch.Tensor, unit_len: List[int],
                 unit_pad: List[int]) -> None:
    """Copy the concatenated unpadded values `src` into `dst` ([psi_pad]) unit
    by unit, zeroing each unit's padding."""
    b = 0
    a = 0
    for n, P in zip(unit_len, unit_pad):
        dst[b:b + n].copy_(src[a:a + n])
        if P > n:
            dst[b + n:b + P].zero_()
        b += P
        a += n


def grad_row(out: torch.Tensor, unit_len: List[int], unit_pad: List[int],
             sigma: float, seed: int, outlier_frac: float = 0.0,
             outlier_scale: float = 100.0) -> torch.Tensor:
    """Fill one rank's bf16 gradient row `out` ([psi_pad], bf16, any device)."""
    dev = out.device
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    psi = sum(unit_len)
    x = torch.randn(psi, generator=g, device=dev, dtype=torch.float32)
    x.mul_(sigma)
    if outlier_frac > 0.0:
        mask = torch.rand(psi, generator=g, device=dev) < outlier_frac
        x = torch.where(mask, x * outlier_scale, x)
    _fill_padded(out, x.to(torch.bfloat16), unit_len, unit_pad)
    return out


def grads(nd: int, unit_len: List[int], unit_pad: List[int], sigma: float,
          config: int, step: int, device, outlier_frac: float = 0.0,
          out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """All Nd ranks' gradients, bf16 [nd, psi_pad]."""
    psi_pad = sum(unit_pad)
    if out is None:
        out = torch.empty((nd, psi_pad), dtype=torch.bfloat16, device=device)
    for r in range(nd):
        grad_row(out[r], unit_len, unit_pad, sigma, seed_for(config, r, step),
                 outlier_frac)
    return out


def master_logical(unit_len: List[int], unit_pad: List[int], config: int,
                   device, std: float = 0.02) -> torch.Tensor:
    """fp32 [psi_pad] master weights in logical order, padding zero."""
    g = torch.Generator(device=device)
    g.manual_seed(master_seed(config))
    psi = sum(unit_len)
    x = torch.randn(psi, generator=g, device=device, dtype=torch.float32)
    x.mul_(std)
    out = torch.empty(sum(unit_pad), dtype=torch.float32, device=device)
    _fill_padded(out, x, unit_len, unit_pad)
    return out
