"""Seeded synthetic inputs for VBQ matrices and activations.

This module only draws random inputs: per-group widths, fp16 scales, codes and bf16 activations. It holds none
of the method's arithmetic (no dequantization, no packing, no products), so both the CUDA path's tests and the
oracle can take their inputs from it.

Workload shapes follow the VBQ paper ("Variable Bit-width Quantization"): the per-group width mix of section 5.1
(about 69% of groups at 1 bit), the first-block MLP kept at about 2.5 bits with about 10% 8-bit groups, and the
language-model head at about 1.09 mean bits with 92.5% of rows pure 1-bit (section 5.1). The trained weights
behind those numbers are not available, so these draws stand in for them.

Seeding: every array comes from ``numpy.random.default_rng(SeedSequence([0, cfg, layer, proj, stream]))``.
proj is q=0, k=1, v=2, o=3, gate=4, up=5, down=6, head=7, single=0. stream is widths=0, scales=1, codes=2,
x=3.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

P_BASE = (0.69, 0.16, 0.09, 0.06)          # P(1,2,4,8 bit) per group, mean 1.85 bits
P_FIRST_MLP = (0.40, 0.35, 0.15, 0.10)     # mean 2.50 bits, 10% 8-bit groups
P_HEAD_TOP = (0.30, 0.45, 0.25, 0.0)       # frequent-token head rows, mean 2.2 bits
WIDTHS = np.array([1, 2, 4, 8], np.uint8)
PROJ = {"single": 0, "q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6, "head": 7}
STREAM = {"widths": 0, "scales": 1, "codes": 2, "x": 3}


def rng(cfg: int, layer: int, proj: str, stream: str) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([0, cfg, layer, PROJ[proj], STREAM[stream]]))


def widths_iid(N: int, G: int, p, g: np.random.Generator) -> np.ndarray:
    return WIDTHS[g.choice(4, size=(N, G), p=np.asarray(p, np.float64))]


def widths_uniform(N: int, G: int, k: int) -> np.ndarray:
    return np.full((N, G), k, np.uint8)


def widths_half_8bit(N: int, G: int, g: np.random.Generator) -> np.ndarray:
    """Exactly G/2 groups per row at 8 bits, the rest 1 bit, positions shuffled per row."""
    w = np.ones((N, G), np.uint8)
    for r in range(N):
        w[r, g.permutation(G)[: G // 2]] = 8
    return w


def widths_head(N: int, G: int, g: np.random.Generator, top: int = 2400, top8: int = 1000,
                frac8: float = 0.048) -> np.ndarray:
    """LM-head widths: rows [0, top) draw from P_HEAD_TOP; a random frac8 of rows [0, top8) get one extra 8-bit
    group; the remaining rows are pure 1-bit (rows are in descending token-frequency order)."""
    w = np.ones((N, G), np.uint8)
    t = min(top, N)
    w[:t] = widths_iid(t, G, P_HEAD_TOP, g)
    t8 = min(top8, N)
    rows = g.choice(t8, size=int(round(frac8 * t8)), replace=False)
    cols = g.integers(0, G, size=rows.size)
    w[rows, cols] = 8
    return w


def scales_uniform(N: int, G: int, g: np.random.Generator, lo: float = 0.01, hi: float = 0.1) -> np.ndarray:
    """fp16 bit patterns of U(lo, hi) draws (round-to-nearest-even float32 -> float16 cast)."""
    return g.uniform(lo, hi, size=(N, G)).astype(np.float32).astype(np.float16).view(np.uint16)


def codes_uniform(widths: np.ndarray, g: np.random.Generator) -> np.ndarray:
    """Uniform codes in [0, 2^k): uniform random bytes masked to the group's k low bits."""
    N, G = widths.shape
    raw = g.integers(0, 256, size=(N, G * 64), dtype=np.uint8)
    mask = ((np.uint16(1) << widths.astype(np.uint16)) - 1).astype(np.uint8)
    return raw & np.repeat(mask, 64, axis=1)


def x_normal(B: int, K: int, g: np.random.Generator) -> np.ndarray:
    """bf16 bit patterns of N(0,1) float32 draws, rounded to nearest even (via torch's cast)."""
    import torch
    x = torch.from_numpy(g.standard_normal(size=(B, K), dtype=np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


@dataclass
class Matrix:
    name: str
    N: int
    K: int
    widths: np.ndarray   # [N, G] uint8 in {1,2,4,8}
    scales: np.ndarray   # [N, G] uint16 fp16 bits
    codes: np.ndarray    # [N, K] uint8

    @property
    def G(self) -> int:
        return self.K // 64


def make_matrix(cfg: int, proj: str, N: int, K: int, widths: np.ndarray | None = None, p=P_BASE,
                layer: int = 0, name: str | None = None) -> Matrix:
    G = K // 64
    if widths is None:
        widths = widths_iid(N, G, p, rng(cfg, layer, proj, "widths"))
    scales = scales_uniform(N, G, rng(cfg, layer, proj, "scales"))
    codes = codes_uniform(widths, rng(cfg, layer, proj, "codes"))
    return Matrix(name or proj, N, K, widths, scales, codes)


def make_x(cfg: int, proj: str, B: int, K: int, layer: int = 0) -> np.ndarray:
    return x_normal(B, K, rng(cfg, layer, proj, "x"))


# ----------------------------------------------------------------------------- workload configurations
def cfg1():
    """Single 768x768 linear (12 groups per row), batch 1, base width mix, seed 0."""
    return [make_matrix(1, "single", 768, 768)]


def cfg2():
    """One 1.0B-shaped decoder layer (d=2048, MLP 5632): q,k,v,o at the base mix; gate, up, down at the
    first-block MLP mix (mean 2.5 bits)."""
    out = [make_matrix(2, p, 2048, 2048) for p in ("q", "k", "v", "o")]
    out += [make_matrix(2, p, 5632, 2048, p=P_FIRST_MLP) for p in ("gate", "up")]
    out.append(make_matrix(2, "down", 2048, 5632, p=P_FIRST_MLP))
    return out


def cfg3(N: int = 4096, K: int = 4096):
    """Uniform-width edge sweep: all-1, all-2, all-4, all-8 bit, and exactly half 8-bit per row."""
    G = K // 64
    out = [make_matrix(3, "single", N, K, widths=widths_uniform(N, G, k), layer=i, name=f"all{k}")
           for i, k in enumerate((1, 2, 4, 8))]
    out.append(make_matrix(3, "single", N, K, widths=widths_half_8bit(N, G, rng(3, 4, "single", "widths")),
                           layer=4, name="mix1_8"))
    return out


CFG4_SHAPES = {"q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
               "gate": (14336, 4096), "up": (14336, 4096), "down": (4096, 14336)}


def cfg4(names=("q", "k", "v", "o", "gate", "up", "down")):
    """9B-shaped linears (d=4096, MLP 14336) at the base width mix; batches 1, 2, 4, 8, 16."""
    return [make_matrix(4, n, *CFG4_SHAPES[n]) for n in names]


def cfg5_layer(layer: int):
    """One layer of the 9B-shaped decode stack (32 layers); layer 0's MLP uses the first-block mix."""
    out = []
    for n in ("q", "k", "v", "o", "gate", "up", "down"):
        N, K = CFG4_SHAPES[n]
        p = P_FIRST_MLP if (layer == 0 and n in ("gate", "up", "down")) else P_BASE
        out.append(make_matrix(5, n, N, K, p=p, layer=layer))
    return out


def cfg5_head(N: int = 32000, K: int = 4096):
    """LM head 4096 -> 32000 at about 1.09 mean bits."""
    return make_matrix(5, "head", N, K, widths=widths_head(N, K // 64, rng(5, 0, "head", "widths")))


# Fixed deployment recipe (VBQ paper, section 3.4): one width per projection instead of per group. The first
# block's MLP stays at 4 bits, every other projection is 2-bit, and the language-model head is tiered by token
# frequency: the top 0.5% of rows (in descending frequency order) 8-bit, the next 1.5% 4-bit, the next 10%
# 2-bit and the remaining 88% 1-bit (mean 0.005*8 + 0.015*4 + 0.10*2 + 0.88*1 = 1.18 bits).
RECIPE_HEAD_TIERS = ((0.005, 8), (0.015, 4), (0.10, 2), (0.88, 1))


def widths_head_tiered(N: int, G: int) -> np.ndarray:
    """Recipe head widths: row tiers in descending token-frequency order (RECIPE_HEAD_TIERS)."""
    w = np.ones((N, G), np.uint8)
    start = 0
    for frac, k in RECIPE_HEAD_TIERS[:-1]:
        stop = min(N, start + int(round(frac * N)))
        w[start:stop] = k
        start = stop
    return w


def cfg6_recipe_layer(layer: int):
    """One 9B-shaped layer under the fixed recipe: MLP (gate, up, down) 4-bit in layer 0, 2-bit elsewhere;
    attention projections 2-bit."""
    out = []
    for n in ("q", "k", "v", "o", "gate", "up", "down"):
        N, K = CFG4_SHAPES[n]
        k = 4 if (layer == 0 and n in ("gate", "up", "down")) else 2
        out.append(make_matrix(6, n, N, K, widths=widths_uniform(N, K // 64, k), layer=layer))
    return out


def cfg6_recipe_head(N: int = 32000, K: int = 4096):
    """LM head 4096 -> 32000 under the recipe's frequency tiers (mean 1.18 bits)."""
    return make_matrix(6, "head", N, K, widths=widths_head_tiered(N, K // 64))


MLP8960 = {"hidden": 1536, "inter": 8960}   # an MLP whose intermediate width is not a multiple of 512


def cfg7_mlp(hidden: int = MLP8960["hidden"], inter: int = MLP8960["inter"]):
    """gate and up (inter x hidden) and down (hidden x inter) at the base width distribution: the shape on which
    the zero-padded packing (intermediate width rounded up to a multiple of 512) is compared with the unpadded
    one."""
    return [make_matrix(7, "gate", inter, hidden), make_matrix(7, "up", inter, hidden),
            make_matrix(7, "down", hidden, inter)]
