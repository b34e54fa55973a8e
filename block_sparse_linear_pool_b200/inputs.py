"""Seeded synthetic inputs for the SLA / SLA2 forward.

This module holds no arithmetic of the method itself: it only draws tensors.
Both the CUDA path and the CPU oracle consume exactly the bf16 tensors it
returns, so the two sides always see the same bits.

Two recipes:

* ``block_mean_inputs`` - Q, K, V = N(0, 1) noise plus a mean vector shared by
  the tokens of each 64-token block, drawn N(0, mean_std^2) independently per
  (tensor, batch, head, block, channel).  The shared mean makes block pooling
  informative.  Used for the tiny case (B=1, H=2, N=1024, d=64).
* ``grid_field_inputs`` - video-shaped activations: N tokens laid out row-major
  on a (t, h, w) grid (token n = (t*Hh + h)*Ww + w).  For every (head, channel)
  the value is a sum of 8 random plane waves
  a*sin(2*pi*(f_t*t/Tt + f_h*h/Hh + f_w*w/Ww) + psi), f ~ U(0, 2) cycles per
  extent, a ~ N(0, 1)/sqrt(8), psi ~ U(0, 2*pi), plus N(0, 1) noise.  Q and K of
  a head are multiplied by one common factor so that the logits q.k/sqrt(d) of
  1e5 random (query, key) pairs have standard deviation ~3.  Seeds: numpy PCG64
  seed 0 for Q, 1 for K, 2 for V, 3 for the parameters.  This stands in for the
  Wan2.1 attention activations the pages measure on, which are not available.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def block_mean_inputs(B=1, H=2, N=1024, d=64, block=64, mean_std=0.5, seed=0,
                      proj_std=0.02):
    """Tiny-case inputs: returns dict(Q, K, V bf16 [B,H,N,d], proj_w fp32 [d,d], proj_b None)."""
    rng = np.random.default_rng(seed)
    T = -(-N // block)
    out = {}
    for name in ("Q", "K", "V"):
        x = rng.standard_normal((B, H, N, d))
        means = rng.standard_normal((B, H, T, d)) * mean_std
        x = x + np.repeat(means, block, axis=2)[:, :, :N, :]
        out[name] = _bf16(x)
    out["proj_w"] = torch.from_numpy(rng.standard_normal((d, d)) * proj_std).float()
    out["proj_b"] = None
    return out


def _grid_coords(grid):
    Tt, Hh, Ww = grid
    n = np.arange(Tt * Hh * Ww)
    t = n // (Hh * Ww)
    h = (n // Ww) % Hh
    w = n % Ww
    return t / Tt, h / Hh, w / Ww


def _wave_field(rng, B, H, d, grid, n_waves, device):
    """sum of n_waves random plane waves + N(0,1) noise, float32 [B,H,N,d]."""
    N = int(np.prod(grid))
    f = rng.uniform(0.0, 2.0, size=(B, H, d, n_waves, 3))
    a = rng.standard_normal((B, H, d, n_waves)) / math.sqrt(n_waves)
    psi = rng.uniform(0.0, 2.0 * math.pi, size=(B, H, d, n_waves))
    noise = rng.standard_normal((B, H, N, d), dtype=np.float32)
    ct, ch, cw = (torch.tensor(c, dtype=torch.float32, device=device) for c in _grid_coords(grid))
    out = torch.empty((B, H, N, d), dtype=torch.float32, device=device)
    for b in range(B):
        for hh in range(H):
            fb = torch.tensor(f[b, hh], dtype=torch.float32, device=device)      # [d, W, 3]
            ab = torch.tensor(a[b, hh], dtype=torch.float32, device=device)      # [d, W]
            pb = torch.tensor(psi[b, hh], dtype=torch.float32, device=device)    # [d, W]
            phase = (fb[..., 0:1] * ct + fb[..., 1:2] * ch + fb[..., 2:3] * cw) * (2 * math.pi)
            phase = phase + pb[..., None]                                        # [d, W, N]
            out[b, hh] = (ab[..., None] * torch.sin(phase)).sum(dim=1).T
    out += torch.from_numpy(noise).to(device)
    return out


def grid_field_inputs(B=1, H=12, d=128, grid=(21, 30, 52), n_waves=8, logit_std=3.0,
                      combine="proj", seeds=(0, 1, 2, 3), device: Optional[str] = None,
                      proj_std=0.02, n_pairs=100_000):
    """Video-grid inputs.  Returns dict with Q, K, V (bf16 [B,H,N,d] on CPU) and the
    parameters of the chosen combine:
      combine="proj":  proj_w fp32 [d,d] ~ N(0, proj_std^2), proj_b None
      combine="alpha": alpha fp32 [B,H] ~ U(0.6, 0.95); Wq, Wk fp32 [d,d] ~ U(-1/sqrt(d), 1/sqrt(d))
    """
    device = device or "cpu"
    N = int(np.prod(grid))
    fields = {}
    for name, s in zip(("Q", "K", "V"), seeds[:3]):
        fields[name] = _wave_field(np.random.default_rng(s), B, H, d, grid, n_waves, device)
    prng = np.random.default_rng(seeds[3])
    # common Q/K factor per head so that std(q.k/sqrt(d)) ~ logit_std
    qi = torch.from_numpy(prng.integers(0, N, size=n_pairs)).to(device)
    ki = torch.from_numpy(prng.integers(0, N, size=n_pairs)).to(device)
    for b in range(B):
        for hh in range(H):
            q = fields["Q"][b, hh][qi]
            k = fields["K"][b, hh][ki]
            std = float(((q * k).sum(-1) / math.sqrt(d)).std())
            c = math.sqrt(logit_std / std) if std > 0 else 1.0
            fields["Q"][b, hh] *= c
            fields["K"][b, hh] *= c
    out = {name: fields[name].to(torch.bfloat16).cpu() for name in ("Q", "K", "V")}
    if combine == "proj":
        out["proj_w"] = torch.from_numpy(prng.standard_normal((d, d)) * proj_std).float()
        out["proj_b"] = None
    elif combine == "alpha":
        out["alpha"] = torch.from_numpy(prng.uniform(0.6, 0.95, size=(B, H))).float()
        lim = 1.0 / math.sqrt(d)
        out["Wq"] = torch.from_numpy(prng.uniform(-lim, lim, size=(d, d))).float()
        out["Wk"] = torch.from_numpy(prng.uniform(-lim, lim, size=(d, d))).float()
    else:
        raise ValueError(combine)
    return out


# The five workloads, by what they are.  Sizes from the pages' Wan2.1 settings.
WORKLOADS = {
    "tiny_sla": dict(kind="block_mean", B=1, H=2, N=1024, d=64, k_h=0.10, k_l=0.60,
                     combine="proj"),
    "wan1.3b_sla": dict(kind="grid", B=1, H=12, d=128, grid=(21, 30, 52), k_h=0.05, k_l=0.75,
                        combine="proj"),
    "wan1.3b_sla2": dict(kind="grid", B=1, H=12, d=128, grid=(21, 30, 52), k_h=0.03,
                         k_l=0.80, combine="alpha"),
    "wan14b_720p_sla2": dict(kind="grid", B=1, H=40, d=128, grid=(21, 45, 80), k_h=0.03,
                             k_l=0.80, combine="alpha"),
}


def make_workload(name: str, device: Optional[str] = None, problem: int = 0, **overrides):
    """Inputs of a named workload (see WORKLOADS) as a dict, plus its settings.

    `problem` selects one of many independent problems of the same shape (seeds
    4p .. 4p+3); problem 0 is the default instance.  Data-parallel runs give each
    rank its own problem."""
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    if cfg["kind"] == "block_mean":
        data = block_mean_inputs(B=cfg["B"], H=cfg["H"], N=cfg["N"], d=cfg["d"], seed=problem)
    else:
        seeds = tuple(4 * problem + i for i in range(4))
        data = grid_field_inputs(B=cfg["B"], H=cfg["H"], d=cfg["d"], grid=cfg["grid"],
                                 combine=cfg["combine"], seeds=seeds, device=device)
        cfg["N"] = int(np.prod(cfg["grid"]))
    return data, cfg
