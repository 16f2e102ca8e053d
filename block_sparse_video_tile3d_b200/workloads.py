"""Seeded synthetic inputs shaped like the attention layers of a video diffusion transformer.

This module holds random draws and fixed block-mask patterns only. It computes no step of the
tile-sparse attention method (no tiling, pooling, scoring, selection or attention): both the CUDA
path and the CPU oracle consume what it returns as plain inputs.

Workload recipe (all tensors are generated on the CPU with ``torch.Generator`` so the values do not
depend on the device; Q, K and V are drawn in fp32 in raster order ``[B, L, heads, D]`` and then
rounded to bf16):

* ``tiny``   B=1, heads=2,  D=64,  grid 4x8x8    (256 tokens),    iid N(0,1),            top-k 2
* ``small``  B=1, heads=12, D=128, grid 16x32x56 (28,672 tokens), N(0,1) + cube offset,   top-k 56
* ``large``  B=1, heads=40, D=128, grid 20x48x80 (76,800 tokens), N(0,1) + cube offset,   top-k 120
* ``bsa``    the ``small`` shape and recipe; query prune at cosine 0.95, KV mass 0.9
* ``ragged_sliding`` / ``ragged_random``  B=2, heads=24, D=128, grid 21x30x52 (32,760 tokens),
  iid N(0,1); a fixed 3x3x3 sliding window of cubes, or a Bernoulli(0.15) block mask per
  (batch, head, query cube, key cube) with the diagonal forced on.

"Cube offset": every 4x4x4 cube of the latent grid gets its own offset vector per (batch, head),
drawn from N(0, 0.5^2) independently for Q, K and V and added to every token of that cube before
the bf16 rounding, so that cubes have distinct means (otherwise mean-pooled scores are all near
zero and tile selection is arbitrary).
"""
from __future__ import annotations

import dataclasses
import math

import torch

CUBE = 4  # edge of the 4x4x4 token cube (64 tokens)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    D: int
    T: int
    H: int
    W: int
    mode: str  # "topk" | "bsa" | "mask"
    seed: int
    offset_std: float = 0.0
    k: int = 0
    cos_thresh: float = 0.95
    mass: float = 0.9
    min_kv: int = 1
    mask: str = ""  # "sliding" | "random" for mode == "mask"
    density: float = 0.15

    @property
    def L(self) -> int:
        return self.T * self.H * self.W

    @property
    def grid_tiles(self) -> tuple[int, int, int]:
        return (math.ceil(self.T / CUBE), math.ceil(self.H / CUBE), math.ceil(self.W / CUBE))

    @property
    def nT(self) -> int:
        a, b, c = self.grid_tiles
        return a * b * c

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 64, 4, 8, 8, "topk", 1000, 0.0, k=2),
    "small": Workload("small", 1, 12, 128, 16, 32, 56, "topk", 1001, 0.5, k=56),
    "large": Workload("large", 1, 40, 128, 20, 48, 80, "topk", 1002, 0.5, k=120),
    "bsa": Workload("bsa", 1, 12, 128, 16, 32, 56, "bsa", 1003, 0.5, cos_thresh=0.95, mass=0.9,
                    min_kv=1),
    "ragged_sliding": Workload("ragged_sliding", 2, 24, 128, 21, 30, 52, "mask", 1004, 0.0,
                               mask="sliding"),
    "ragged_random": Workload("ragged_random", 2, 24, 128, 21, 30, 52, "mask", 1004, 0.0,
                              mask="random", density=0.15),
}


def _cube_field(gen: torch.Generator, B: int, T: int, H: int, W: int, heads: int, D: int,
                std: float) -> torch.Tensor:
    """One N(0, std^2) vector per (batch, 4x4x4 cube, head), broadcast to the cube's tokens.

    Returns ``[B, T, H, W, heads, D]`` fp32 (piecewise constant over cubes, cropped at the grid edge).
    """
    nt, nh, nw = (math.ceil(T / CUBE), math.ceil(H / CUBE), math.ceil(W / CUBE))
    vec = torch.randn((B, nt, nh, nw, heads, D), generator=gen, dtype=torch.float32) * std
    vec = vec.repeat_interleave(CUBE, 1).repeat_interleave(CUBE, 2).repeat_interleave(CUBE, 3)
    return vec[:, :T, :H, :W]


def make_qkv(w: Workload, seed: int | None = None):
    """Q, K, V as bf16 CPU tensors ``[B, L, heads, D]`` in raster (t, h, w) token order."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    out = []
    for _ in range(3):
        x = torch.randn((w.B, w.T, w.H, w.W, w.heads, w.D), generator=gen, dtype=torch.float32)
        if w.offset_std > 0:
            x += _cube_field(gen, w.B, w.T, w.H, w.W, w.heads, w.D, w.offset_std)
        out.append(x.reshape(w.B, w.L, w.heads, w.D).to(torch.bfloat16))
    return tuple(out)


def make_structured_queries(w: Workload, q: torch.Tensor, seed: int | None = None,
                            frac: float = 0.5, noise: float = 0.05) -> torch.Tensor:
    """Query variant with redundant tokens: in a seeded ``frac`` of the (batch, cube, head) cells
    every token is the cube's own random vector plus N(0, noise^2), so that query pruning by cosine
    similarity has rows to drop. Other cells keep ``q``. Returns bf16 ``[B, L, heads, D]``."""
    gen = torch.Generator().manual_seed((w.seed if seed is None else seed) + 7919)
    nt, nh, nw = w.grid_tiles
    pick = (torch.rand((w.B, nt, nh, nw, w.heads), generator=gen) < frac).to(torch.float32)
    pick = pick.repeat_interleave(CUBE, 1).repeat_interleave(CUBE, 2).repeat_interleave(CUBE, 3)
    pick = pick[:, :w.T, :w.H, :w.W].unsqueeze(-1)
    base = _cube_field(gen, w.B, w.T, w.H, w.W, w.heads, w.D, 1.0)
    red = base + noise * torch.randn(base.shape, generator=gen, dtype=torch.float32)
    qf = q.reshape(w.B, w.T, w.H, w.W, w.heads, w.D).to(torch.float32)
    qs = pick * red + (1.0 - pick) * qf
    return qs.reshape(w.B, w.L, w.heads, w.D).to(torch.bfloat16)


def sliding_cube_mask(nt: int, nh: int, nw: int, radius: int = 1) -> torch.Tensor:
    """Fixed sliding-window block mask over the cube grid: query cube i keeps key cube j iff their
    cube coordinates differ by at most ``radius`` along t, h and w. The window is clipped at the
    grid edge (not shifted inward), so a row keeps between 8 and 27 cubes for radius 1.

    Cubes are numbered t-major, then h, then w. Returns uint8 ``[nT, nT]``."""
    ct = torch.arange(nt).view(nt, 1, 1).expand(nt, nh, nw).reshape(-1)
    ch = torch.arange(nh).view(1, nh, 1).expand(nt, nh, nw).reshape(-1)
    cw = torch.arange(nw).view(1, 1, nw).expand(nt, nh, nw).reshape(-1)
    near = ((ct[:, None] - ct[None, :]).abs() <= radius) & \
           ((ch[:, None] - ch[None, :]).abs() <= radius) & \
           ((cw[:, None] - cw[None, :]).abs() <= radius)
    return near.to(torch.uint8)


def random_block_mask(B: int, heads: int, nT: int, density: float, seed: int) -> torch.Tensor:
    """Bernoulli(``density``) block mask per (batch, head, query cube, key cube) with the diagonal
    forced on (so every query cube keeps at least one key cube). Returns uint8 ``[B, heads, nT, nT]``."""
    gen = torch.Generator().manual_seed(seed)
    m = torch.rand((B, heads, nT, nT), generator=gen) < density
    idx = torch.arange(nT)
    m[:, :, idx, idx] = True
    return m.to(torch.uint8)


def block_mask(w: Workload) -> torch.Tensor:
    """The fixed block mask of a ``mask``-mode workload, as uint8 ``[B, heads, nT, nT]``."""
    if w.mask == "sliding":
        m = sliding_cube_mask(*w.grid_tiles)
        return m.view(1, 1, w.nT, w.nT).expand(w.B, w.heads, w.nT, w.nT).contiguous()
    if w.mask == "random":
        return random_block_mask(w.B, w.heads, w.nT, w.density, w.seed)
    raise ValueError(f"workload {w.name} has no fixed block mask")


# ------------------------------------------------------------------ packed multi-region sequences

@dataclasses.dataclass(frozen=True)
class PackedWorkload:
    """A packed sequence (video_sparse_attn_h3 page, build()): dense segments (row counts) and
    video regions (token grids, patch 1), the last region the generated video."""
    name: str
    B: int
    heads: int
    D: int
    segments: tuple
    tile_size: int
    sparsity: float
    ref_keep_rate: float
    seed: int


PACKED_WORKLOADS = {
    # a text prefix, one reference clip at half the frames and the generated clip of the small
    # layer's grid, with 128-token tiles
    "packed": PackedWorkload("packed", 1, 12, 128, (512, (8, 32, 56), (16, 32, 56)), 128, 0.875,
                             0.25, 1005),
    "packed_tiny": PackedWorkload("packed_tiny", 1, 2, 64, (37, (4, 8, 8), (5, 8, 12)), 128, 0.75,
                                  0.5, 1006),
}


def packed_rows(w: PackedWorkload) -> int:
    return sum(s if isinstance(s, int) else s[0] * s[1] * s[2] for s in w.segments)


def make_packed_qkv(w: PackedWorkload, seed: int | None = None):
    """Q, K, V as bf16 CPU tensors ``[B, rows, heads, D]`` in packed order: i.i.d. N(0, 1) (the
    region structure only sets where the tiles lie)."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    shape = (w.B, packed_rows(w), w.heads, w.D)
    return tuple(torch.randn(shape, generator=g).to(torch.bfloat16) for _ in range(3))
