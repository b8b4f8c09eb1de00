"""Seeded synthetic workloads for the Veda tile-skipping attention layer.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests. It holds only workload descriptions (grid, heads, head dim, tile size,
per-head tilings, keep fraction, seed) and random-number generation. It holds
none of the method's arithmetic: no permutation, pooling, scoring, top-k or
attention happens here.

Workloads follow the shapes of the 720P video DiT layers that the Veda pages
("Technical Summary: Veda - Scalable Video Diffusion via Distilled Sparse
Attention", section 4) measure on. Model activations are not available, so
Q and K are Gaussian noise plus a 3-D sinusoidal position term, which makes
attention spatio-temporally local (the head-dependent locality of section 2.2),
and V is Gaussian noise.

Readings of unstated details (all recorded in the design notes):
  * position features: per axis D_a = 2*floor(d/6) dims laid out as
    [sin | cos] of coord * 10000**(-2i/D_a), axes in (t, h, w) order, the rest
    of the head dim zero;
  * q, k = 0.5*N(0,1) + 1.5*pos (independent noise per tensor and head),
    v ~ N(0,1); everything rounded to bf16 (round to nearest even);
  * tile scorer: one MLP per head, Linear(3d,128) -> GELU -> Linear(128,64),
    Xavier-uniform weights, zero biases, applied to both Q and K descriptors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

Tiling = Tuple[int, int, int]

TILINGS_64: Tuple[Tiling, ...] = ((1, 8, 8), (2, 4, 8), (4, 4, 4), (4, 2, 8))
TILINGS_128: Tuple[Tiling, ...] = ((2, 8, 8), (1, 8, 16), (4, 4, 8), (8, 4, 4))

MLP_HIDDEN = 128
MLP_OUT = 64
SCORE_SCALE = 1.0 / 8.0


@dataclass(frozen=True)
class Workload:
    """One synthetic attention layer: B x (T*H*W) tokens x heads x d."""
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    tile: int
    tilings: Tuple[Tiling, ...]          # one per head
    keep: float                          # fraction of key tiles kept per row
    seed: int
    tilemap_heads: Tuple[int, ...] = ()  # heads whose full-attention tile map is built
    tilemap_rows: Optional[int] = None   # query tiles per tile-map head (None = all)
    k_fixed: Optional[int] = None        # explicit k (overrides keep) for tiny cases

    @property
    def N(self) -> int:
        return self.T * self.H * self.W


def _draw_tilings(rng: np.random.Generator, choices: Sequence[Tiling], heads: int) -> Tuple[Tiling, ...]:
    pick = rng.integers(0, len(choices), size=heads)
    return tuple(tuple(int(v) for v in choices[i]) for i in pick)


def config(idx: int, keep: Optional[float] = None) -> Workload:
    """The five named workloads (0: tiny, 1: 24k tokens, 2: 720P-5s-like,
    3: 720P-10s-like, 4: one head group at 64k tokens; see ``sweep`` for the
    full token-count sweep)."""
    if idx == 0:
        return Workload("tiny-256tok-2h-d64", 1, 2, 64, 4, 8, 8, 64,
                        ((1, 8, 8), (4, 4, 4)), 0.5, 0, tilemap_heads=(0, 1), k_fixed=2)
    if idx == 1:
        rng = np.random.default_rng(1 + 1000)
        return Workload("grid16x32x48-24576tok-12h-d128", 1, 12, 128, 16, 32, 48, 64,
                        _draw_tilings(rng, TILINGS_64, 12), 0.2 if keep is None else keep, 1,
                        tilemap_heads=(0, 5))
    if idx == 2:
        rng = np.random.default_rng(2 + 1000)
        return Workload("720p5s-grid21x48x80-80640tok-40h-d128", 1, 40, 128, 21, 48, 80, 128,
                        _draw_tilings(rng, TILINGS_128, 40), 0.1 if keep is None else keep, 2,
                        tilemap_heads=(0, 1))
    if idx == 3:
        rng = np.random.default_rng(3 + 1000)
        tilings = _draw_tilings(rng, TILINGS_128, 24)
        heads = tuple(sorted(int(h) for h in rng.choice(24, size=2, replace=False)))
        return Workload("720p10s-grid40x48x80-153600tok-24h-d128", 1, 24, 128, 40, 48, 80, 128,
                        tilings, 0.1 if keep is None else keep, 3, tilemap_heads=heads)
    if idx == 4:
        return sweep(65280, 0.1)
    raise ValueError(f"no workload {idx}")


SWEEP_TOKENS = (15360, 34560, 65280, 130560, 261120)
SWEEP_KEEP = (1.0, 0.5, 0.2, 0.1, 0.05, 0.03)


def sweep(tokens: int, keep: float) -> Workload:
    """One point of the head-group sweep: 8 heads, d=128, tile=128, grid
    T x 48 x 80 with T = round(tokens/3840); tilings drawn from the 128-token
    set restricted to p_t | T, (1,8,16) always allowed, so no tile is padded."""
    T = int(round(tokens / 3840))
    allowed = tuple(t for t in TILINGS_128 if T % t[0] == 0 or t == (1, 8, 16))
    rng = np.random.default_rng(4 + 1000 + T)
    return Workload(f"sweep-grid{T}x48x80-{T*3840}tok-8h-d128-keep{keep:g}", 1, 8, 128, T, 48, 80, 128,
                    _draw_tilings(rng, allowed, 8), keep, 4, tilemap_heads=(0,))


def custom(name: str, B: int, heads: int, d: int, T: int, H: int, W: int, tile: int,
           tilings: Sequence[Tiling], keep: float, seed: int, k_fixed: Optional[int] = None,
           tilemap_heads: Sequence[int] = ()) -> Workload:
    return Workload(name, B, heads, d, T, H, W, tile, tuple(tuple(t) for t in tilings), keep, seed,
                    tilemap_heads=tuple(tilemap_heads), k_fixed=k_fixed)


def head_subset(w: Workload, h0: int, h1: int) -> Workload:
    """The same layer restricted to heads [h0, h1): their tilings, and the
    tile-map heads among them renumbered from 0. The tensors and weights of
    the subset are the full layer's (slice qkv() and mlp_weights() by head);
    the seed stays the full layer's."""
    if not (0 <= h0 < h1 <= w.heads):
        raise ValueError(f"head range [{h0}, {h1}) outside [0, {w.heads})")
    return replace(w, name=f"{w.name}-heads{h0}-{h1}", heads=h1 - h0, tilings=w.tilings[h0:h1],
                   tilemap_heads=tuple(h - h0 for h in w.tilemap_heads if h0 <= h < h1))


# ---------------------------------------------------------------------------
# random tensors
# ---------------------------------------------------------------------------

def position_features(T: int, H: int, W: int, d: int, device="cpu") -> torch.Tensor:
    """[T*H*W, d] fp32 sinusoidal 3-D position features (token order
    n = (t*H + y)*W + x)."""
    Da = 2 * (d // 6)
    half = Da // 2
    i = torch.arange(half, dtype=torch.float64, device=device)
    freq = torch.pow(torch.tensor(10000.0, dtype=torch.float64, device=device), -2.0 * i / Da)
    feats = []
    for n_axis, (size, rep_before, rep_after) in enumerate(((T, 1, H * W), (H, T, W), (W, T * H, 1))):
        c = torch.arange(size, dtype=torch.float64, device=device)
        ang = c[:, None] * freq[None, :]
        blk = torch.cat([torch.sin(ang), torch.cos(ang)], dim=1)          # [size, Da]
        blk = blk[None, :, None, :].expand(rep_before, size, rep_after, Da).reshape(-1, Da)
        feats.append(blk)
    pos = torch.zeros(T * H * W, d, dtype=torch.float64, device=device)
    pos[:, : 3 * Da] = torch.cat(feats, dim=1)
    return pos.float()


def qkv(w: Workload, device="cpu", seed_offset: int = 0):
    """Q, K, V as [B, N, heads, d] bf16 on ``device`` (seeded generator of
    that device; a given (workload, device) pair always gives the same
    tensors)."""
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * (w.seed + 1) + seed_offset)
    shape = (w.B, w.N, w.heads, w.d)
    pos = position_features(w.T, w.H, w.W, w.d, device=device)[None, :, None, :]
    out = []
    for name in ("q", "k", "v"):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if name != "v":
            x.mul_(0.5).add_(pos, alpha=1.5)
        out.append(x.to(torch.bfloat16))
        del x
    return tuple(out)


def mlp_weights(w: Workload, hidden: int = MLP_HIDDEN, out_dim: int = MLP_OUT):
    """Per-head scorer weights (fp32, numpy): w1 [heads,3d,hidden], b1
    [heads,hidden], w2 [heads,hidden,out], b2 [heads,out]; Xavier-uniform
    weights, zero biases."""
    rng = np.random.default_rng(7_000 + w.seed)
    fin = 3 * w.d
    a1 = math.sqrt(6.0 / (fin + hidden))
    a2 = math.sqrt(6.0 / (hidden + out_dim))
    w1 = rng.uniform(-a1, a1, size=(w.heads, fin, hidden)).astype(np.float32)
    w2 = rng.uniform(-a2, a2, size=(w.heads, hidden, out_dim)).astype(np.float32)
    b1 = np.zeros((w.heads, hidden), np.float32)
    b2 = np.zeros((w.heads, out_dim), np.float32)
    return w1, b1, w2, b2


def sample_rows(n_tiles: int, count: int, seed: int) -> np.ndarray:
    """Seeded sample of query-tile rows; always holds the first and last
    tile (the last one carries the padding when an axis does not divide)."""
    if count >= n_tiles:
        return np.arange(n_tiles, dtype=np.int32)
    rng = np.random.default_rng(9_000 + seed)
    mid = rng.choice(np.arange(1, n_tiles - 1), size=count - 2, replace=False)
    return np.sort(np.concatenate([[0, n_tiles - 1], mid])).astype(np.int32)


def random_index_lists(n_rows: int, n_tiles: int, k: int, k_cap: int, seed: int) -> np.ndarray:
    """Random ascending key-tile lists [n_rows, k_cap] (-1 padded): an
    attention input that does not depend on any scorer."""
    rng = np.random.default_rng(11_000 + seed)
    out = np.full((n_rows, k_cap), -1, np.int32)
    for r in range(n_rows):
        out[r, :k] = np.sort(rng.choice(n_tiles, size=k, replace=False))
    return out
