"""Seeded synthetic inputs for the hybrid global-attention layer.

This module is shared by the tests, ``bench.py`` and ``__graft_entry__``: it
produces the bf16 Q/K/V tensors that both the CUDA path and the fp64 oracle
consume.  It holds none of the method's arithmetic (no pooling, scoring,
softmax, feature map or fit) -- only random numbers and the planted structure
of the workloads.

Workloads (shapes follow VGGT-style global attention: 1,374 tokens per view =
37x37 patch tokens + 5 camera/register tokens, 16 heads, head dim 64):

==========  =====  ===========  ====  =====  ==========================
name        heads  tokens       tile  k      planted key tiles per q-tile
==========  =====  ===========  ====  =====  ==========================
tiny        2      4x64 = 256   64    2      1, uniform
views32     16     32 views     128   69     3-5, uniform
linear256   16     256 views    128   --     none (linear stage)
stack512    16     512 views    128   1100   3-5, uniform (per layer)
views1024   16     1,024 views  128   660    3-5, within +-2 views
spatial32   16     32 views     128   69     none; 2-D positional locality
==========  =====  ===========  ====  =====  ==========================

Planting recipe (one reading of "each query tile shares a unit direction with
its hot key tiles"): for every (head h, query tile i) draw a unit vector
u[h,i] (normalised N(0, I_d) in fp32) and m in {lo..hi} distinct key tiles
P(h,i).  Every query row of tile i gets ``2.0 * u[h,i]`` added; every key row
of each tile j in P(h,i) gets ``2.0 * u[h,i]`` added (a key tile that is hot
for several query tiles accumulates several directions).  Values are drawn in
fp32 and rounded once to bf16 (round-to-nearest-even).

Seeds: ``seed = 1000 * config_number + 10 * layer`` unless given.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np
import torch

TOKENS_PER_VIEW = 37 * 37 + 5  # 1,374


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int
    heads: int
    n_tokens: int
    head_dim: int = 64
    tile: int = 128
    keep_frac: Optional[float] = None   # fraction of key tiles kept (sparse stage)
    k_fixed: Optional[int] = None       # explicit k (tiny case)
    v_std: float = 1.0                  # V ~ N(0, v_std^2)
    plant_lo: int = 0                   # planted key tiles per query tile: lo..hi
    plant_hi: int = 0
    plant_window: Optional[int] = None  # +-window (in tiles) around the query tile
    plant_scale: float = 2.0
    calib_tiles: Optional[int] = 32     # calibration query tiles for the affine fit
    layers: int = 1
    linear_layers: Tuple[int, ...] = ()
    pos_scale: float = 0.0              # 2-D positional component of patch-token queries and keys
    pos_length: float = 3.0             # its length scale, in patches

    @property
    def n_tiles(self) -> int:
        return -(-self.n_tokens // self.tile)

    @property
    def k(self) -> Optional[int]:
        if self.k_fixed is not None:
            return self.k_fixed
        if self.keep_frac is None:
            return None
        # budget rounding: k = ceil(frac * T), computed in exact rational arithmetic
        num, den = _as_fraction(self.keep_frac)
        return min(self.n_tiles, -(-(num * self.n_tiles) // den))


def _as_fraction(x: float) -> Tuple[int, int]:
    from fractions import Fraction
    f = Fraction(str(x))
    return f.numerator, f.denominator


WORKLOADS = {
    "tiny": Workload("tiny", 1, heads=2, n_tokens=256, tile=64, k_fixed=2,
                     v_std=1.0 / 8.0, plant_lo=1, plant_hi=1, calib_tiles=None),
    "views32": Workload("views32", 2, heads=16, n_tokens=32 * TOKENS_PER_VIEW,
                        keep_frac=0.20, v_std=1.0, plant_lo=3, plant_hi=5),
    "linear256": Workload("linear256", 3, heads=16, n_tokens=256 * TOKENS_PER_VIEW,
                          v_std=1.0 / 8.0),
    "stack512": Workload("stack512", 4, heads=16, n_tokens=512 * TOKENS_PER_VIEW,
                         keep_frac=0.20, v_std=1.0, plant_lo=3, plant_hi=5, layers=24,
                         linear_layers=(1, 2, 3, 4, 5, 6, 8, 18, 20, 21, 22, 23)),
    "views1024": Workload("views1024", 5, heads=16, n_tokens=1024 * TOKENS_PER_VIEW,
                          keep_frac=0.06, v_std=1.0, plant_lo=3, plant_hi=5,
                          plant_window=22),
    "spatial32": Workload("spatial32", 6, heads=16, n_tokens=32 * TOKENS_PER_VIEW,
                          keep_frac=0.20, v_std=1.0, pos_scale=8.0, pos_length=3.0),
}
GRID = 37        # patches per side of a view
SPECIALS = 5     # camera/register tokens at the start of each view


def default_seed(w: Workload, layer: int = 0) -> int:
    return 1000 * w.number + 10 * layer


def _floyd_sample(rng: np.random.Generator, width: np.ndarray, m: int) -> np.ndarray:
    """m distinct uniform picks from [0, width[r]) for every row r (Floyd's method).

    ``width`` is an int64 array of per-row range sizes, each >= m.
    Returns int64 [rows, m].
    """
    rows = width.shape[0]
    out = np.empty((rows, m), dtype=np.int64)
    for step in range(m):
        top = width - m + step                      # inclusive upper bound this step
        r = np.floor(rng.random(rows) * (top + 1)).astype(np.int64)
        r = np.minimum(r, top)
        if step:
            dup = (out[:, :step] == r[:, None]).any(axis=1)
            r = np.where(dup, top, r)
        out[:, step] = r
    return out


def planted_pairs(w: Workload, seed: int):
    """The planted (head, query tile, key tile) triples, as int64 numpy arrays."""
    if w.plant_hi <= 0:
        z = np.zeros(0, dtype=np.int64)
        return z, z, z
    rng = np.random.default_rng(seed)
    H, T = w.heads, w.n_tiles
    rows = H * T
    m_row = rng.integers(w.plant_lo, w.plant_hi + 1, size=rows)
    if w.plant_window is None:
        lo = np.zeros(rows, dtype=np.int64)
        width = np.full(rows, T, dtype=np.int64)
    else:
        i = np.tile(np.arange(T, dtype=np.int64), H)
        lo = np.maximum(0, i - w.plant_window)
        hi = np.minimum(T - 1, i + w.plant_window)
        width = hi - lo + 1
    if (width < w.plant_hi).any():
        raise ValueError("planting window narrower than the number of planted tiles")
    picks = _floyd_sample(rng, width, w.plant_hi) + lo[:, None]
    keep = np.arange(w.plant_hi)[None, :] < m_row[:, None]
    r_idx, c_idx = np.nonzero(keep)
    h = r_idx // T
    i = r_idx % T
    j = picks[r_idx, c_idx]
    return h.astype(np.int64), i.astype(np.int64), j.astype(np.int64)


def make_qkv(w: Workload, layer: int = 0, device="cpu", seed: Optional[int] = None,
             n_tokens: Optional[int] = None):
    """Q, K, V as bf16 tensors [heads, n_tokens, head_dim] on ``device``.

    ``n_tokens`` overrides the workload's token count (same recipe, other size).
    """
    if seed is None:
        seed = default_seed(w, layer)
    if n_tokens is not None and n_tokens != w.n_tokens:
        w = dataclasses.replace(w, n_tokens=n_tokens)
    H, N, d, t, T = w.heads, w.n_tokens, w.head_dim, w.tile, w.n_tiles
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    inv = 1.0 / math.sqrt(d)
    Q = torch.randn(H, N, d, generator=g, device=dev, dtype=torch.float32).mul_(inv)
    K = torch.randn(H, N, d, generator=g, device=dev, dtype=torch.float32).mul_(inv)
    V = torch.randn(H, N, d, generator=g, device=dev, dtype=torch.float32).mul_(w.v_std)
    if w.plant_hi > 0:
        U = torch.randn(H, T, d, generator=g, device=dev, dtype=torch.float32)
        U = U / U.norm(dim=-1, keepdim=True)
        hh, ii, jj = planted_pairs(w, seed)
        row_tile = torch.arange(N, device=dev) // t
        Q.add_(w.plant_scale * U[:, row_tile, :])
        # accumulate the key-side directions on the host: np.add.at sums in a
        # fixed order, so the inputs are reproducible bit for bit
        u_host = U.to("cpu").numpy()
        kadd = np.zeros((H * T, d), dtype=np.float32)
        np.add.at(kadd, hh * T + jj, np.float32(w.plant_scale) * u_host[hh, ii, :])
        kadd_t = torch.from_numpy(kadd).to(dev)
        K.add_(kadd_t.view(H, T, d)[:, row_tile, :])
        del u_host, kadd, kadd_t
        del U, row_tile
    if w.pos_scale > 0:
        # 2-D locality: patch (y, x) of every view gets pos_scale * E(y, x) added to
        # its query and key, E_c = sqrt(2/d) cos(w_c . (y, x) + phi_c) with per-head
        # random w_c ~ N(0, I / pos_length^2), phi_c ~ U(0, 2 pi): random Fourier
        # features, so E(p) . E(p') approximates exp(-|p - p'|^2 / (2 pos_length^2))
        # and nearby patches (in any view) attend to each other
        per_view = SPECIALS + GRID * GRID
        if N % per_view:
            raise ValueError("positional planting needs whole views")
        om = torch.randn(H, d, 2, generator=g, device=dev, dtype=torch.float32) / w.pos_length
        phi = torch.rand(H, d, generator=g, device=dev, dtype=torch.float32) * (2 * math.pi)
        yy, xx = torch.meshgrid(torch.arange(GRID, device=dev, dtype=torch.float32),
                                torch.arange(GRID, device=dev, dtype=torch.float32), indexing="ij")
        pos = torch.stack([yy.reshape(-1), xx.reshape(-1)], dim=-1)                   # [P, 2]
        E = math.sqrt(2.0 / d) * torch.cos(torch.einsum("pk,hck->hpc", pos, om) + phi[:, None, :])
        add = torch.zeros(H, per_view, d, device=dev, dtype=torch.float32)
        add[:, SPECIALS:] = w.pos_scale * E
        add = add.repeat(1, N // per_view, 1)
        Q.add_(add)
        K.add_(add)
        del add, E
    return (Q.to(torch.bfloat16), K.to(torch.bfloat16), V.to(torch.bfloat16))


def calibration_tiles(n_tiles: int, count: Optional[int]) -> np.ndarray:
    """Whole query tiles used as affine-fit calibration rows: floor(m*T/count), m < count.

    ``count=None`` (or count >= T) means every tile.
    """
    if count is None or count >= n_tiles:
        return np.arange(n_tiles, dtype=np.int64)
    return (np.arange(count, dtype=np.int64) * n_tiles) // count


def to_f64(x: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 (or fp32) tensor to an fp64 numpy array."""
    return x.detach().to("cpu").to(torch.float64).numpy()


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """The raw uint16 bit patterns of a bf16 tensor (host copy)."""
    return x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
