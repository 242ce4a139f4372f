"""Seeded synthetic inputs shared by the CPU oracle side and the CUDA side.

This module only draws random numbers and rounds them to bf16; it holds none
of the reduced-matrix-multiplication arithmetic (no scoring, no selection, no
products).  Both sides of every parity test receive byte-identical bf16
buffers produced here.

Recipe (stand-ins for the trained 1B-70B models the pages evaluate on; no
weights or datasets are used):

* activations X [T, H]: N(0, 1), with a seeded 2 % of the channels
  (``round(0.02 * H)`` columns, chosen by a seeded permutation) scaled by 20
  before rounding -- the outlier-channel structure of LLM activations;
* weights W [N, H]: N(0, std^2) with std = 1/sqrt(H) for the small single-linear
  case and 0.02 for the Llama-shaped projections;
* Q / K / V: N(0, 1);
* tie-heavy inputs: small integers, exact in bf16, so many magnitudes tie.

Values are drawn in fp32 with ``torch.Generator`` on the CPU and rounded to
bf16 with round-to-nearest-even.  Seeds follow ``1000*config + 10*case + stream``.
``device="cuda"`` draws the same recipe with the device's generator instead
(other numbers, same distribution): the benchmark's large workloads use it so
that gigabytes of weights are not drawn on the host; parity tests use the CPU
draws so that both sides see identical bytes.
"""
from __future__ import annotations

import math

import torch

__all__ = [
    "seed_for",
    "activations",
    "weights",
    "normal",
    "tie_heavy",
    "bf16_bits",
]


def seed_for(config: int, case: int, stream: int) -> int:
    """Seed of one input stream of one test case: ``1000*config + 10*case + stream``."""
    return 1000 * int(config) + 10 * int(case) + int(stream)


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(T: int, H: int, seed: int, outlier_frac: float = 0.02,
                outlier_scale: float = 20.0, device="cpu") -> torch.Tensor:
    """X [T, H] bf16: N(0,1) with ``round(outlier_frac*H)`` seeded outlier columns x ``outlier_scale``."""
    g = _gen(seed, device)
    x = torch.randn(T, H, generator=g, dtype=torch.float32, device=device)
    n_out = int(round(outlier_frac * H))
    if n_out > 0:
        cols = torch.randperm(H, generator=g, device=device)[:n_out]
        x[:, cols] *= outlier_scale
    return x.to(torch.bfloat16)


def weights(N: int, H: int, seed: int, std: float | None = None, device="cpu") -> torch.Tensor:
    """W [N, H] bf16 ~ N(0, std^2); ``std=None`` means 1/sqrt(H)."""
    g = _gen(seed, device)
    s = (1.0 / math.sqrt(H)) if std is None else float(std)
    w = torch.randn(N, H, generator=g, dtype=torch.float32, device=device) * s
    return w.to(torch.bfloat16)


def normal(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """A bf16 tensor of the given shape ~ N(0, std^2)."""
    g = _gen(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def tie_heavy(shape, seed: int, lo: int = -3, hi: int = 3) -> torch.Tensor:
    """Small integers in [lo, hi] (exact in bf16): many equal magnitudes, including +0 and -0."""
    g = _gen(seed)
    v = torch.randint(lo, hi + 1, tuple(shape), generator=g).to(torch.float32)
    # flip the sign of some zeros so that -0 and +0 both occur
    flip = torch.rand(tuple(shape), generator=g) < 0.5
    v = torch.where((v == 0) & flip, torch.full_like(v, -0.0), v)
    return v.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """The raw uint16 bit patterns of a bf16 CPU tensor, as a contiguous numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
