"""Seeded synthetic inputs for Skiparse-2D attention.

This module is the only code shared by the CPU oracle's tests and the CUDA path's
tests and benchmark. It holds workload shapes and a seeded random-number recipe and
nothing of the method's arithmetic: no class maps, no padding rule, no attention.

Recipe (stated once, used everywhere): q, k and v are i.i.d. N(0, 1) draws in float32
from ``torch.Generator('cpu').manual_seed(seed)`` via ``torch.randn``, rounded to
bfloat16 with round-to-nearest-even (``.to(torch.bfloat16)``). The layout is
(B, T, H, W, heads, d), contiguous. Seeds: q -> 1000*cfg + 0, k -> 1000*cfg + 1,
v -> 1000*cfg + 2, where ``cfg`` is the workload's family index below.

The shapes stand in for the latent videos of the pages on OSP-Next (5 s clips at
720P and 768P, 81 frames; the summary page's limitations section gives 720x1280 and
81 frames). The latent sizes, heads = 40 and d = 128 are those of a Wan2.1-14B-class
DiT at those resolutions; the pages themselves do not print them.
"""

from __future__ import annotations

import dataclasses

import torch

TOKEN_WISE = 0
GROUP_WISE = 1
MODES = (TOKEN_WISE, GROUP_WISE)
MODE_NAMES = {TOKEN_WISE: "token-wise", GROUP_WISE: "group-wise"}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    family: int  # seed family index
    B: int
    T: int
    H: int
    W: int
    heads: int
    d: int
    P: int

    @property
    def shape(self) -> tuple:
        return (self.B, self.T, self.H, self.W, self.heads, self.d)

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n

    def with_p(self, P: int) -> "Workload":
        return dataclasses.replace(self, P=P, name=f"{self.name.split('_p')[0]}_p{P}")


# Families 0..4: tiny, any-resolution padding, 480p, 720p, 768p latents.
WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 2, 8, 8, 2, 32, 2),
    "anyres": Workload("anyres", 1, 1, 3, 10, 14, 4, 64, 2),
    "480p": Workload("480p", 2, 1, 21, 30, 52, 12, 128, 2),
    "720p": Workload("720p", 3, 1, 21, 45, 80, 40, 128, 2),
    "768p": Workload("768p", 4, 1, 21, 48, 84, 40, 128, 2),
    "768p_p3": Workload("768p_p3", 4, 1, 21, 48, 84, 40, 128, 3),
    "768p_p1": Workload("768p_p1", 4, 1, 21, 48, 84, 40, 128, 1),
}


def randn_bf16(shape, seed: int) -> torch.Tensor:
    """N(0,1) float32 draws from a seeded CPU generator, rounded to bfloat16 (RNE)."""
    g = torch.Generator("cpu")
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(torch.bfloat16)


def qkv(w: Workload, seed_family: int | None = None):
    """The (q, k, v) bfloat16 CPU tensors of a workload, in (B,T,H,W,heads,d) layout."""
    fam = w.family if seed_family is None else seed_family
    return tuple(randn_bf16(w.shape, 1000 * fam + i) for i in range(3))


def custom(B, T, H, W, heads, d, P, name="custom", family=99) -> Workload:
    return Workload(name, family, B, T, H, W, heads, d, P)
