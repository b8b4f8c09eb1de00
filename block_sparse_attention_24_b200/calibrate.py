"""Head-aware tiling search on calibration inputs (Veda summary 2.2: each
head gets the tiling, from a candidate set, that fits its spatio-temporal
locality; the choice is made offline).

For every candidate tiling, applied to all heads at once, the library's own
calls build the oracle tile map of every query tile, keep each row's top-k
key tiles of that map, run the tile-skipping attention with that mask and
measure, per head, its squared distance from full attention (the library's
dense path). A head's tiling is the candidate with the smallest distance.
Only marshalling happens here: every step is a libveda kernel.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import torch

from . import (Layer, veda_check_status, veda_full_attn_tilemax, veda_output_sq_error, veda_permute,
               veda_sparse_attn, veda_topk_mask)
from .layer import k_from_keep

Tiling = Tuple[int, int, int]


def tiling_errors(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, T: int, H: int, W: int, tile: int,
                  candidates: Sequence[Tiling], keep: float, scale: float = None) -> torch.Tensor:
    """q, k, v: [1, N, heads, d] bf16 on the device. Returns errors
    [len(candidates), heads] (fp32, on the host): squared Frobenius distance
    per head between full attention and tile-map-masked sparse attention
    under each candidate tiling."""
    B, N, Hh, d = q.shape
    if B != 1:
        raise ValueError("calibration layers have B == 1")
    dev = q.device
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    # rows padded to 16 bytes: each row is a separately aligned output
    errors = torch.empty((len(candidates), (Hh + 3) // 4 * 4), dtype=torch.float32, device=dev)
    o_full = None
    for c, tiling in enumerate(candidates):
        L = Layer(1, Hh, d, T, H, W, tile, [tuple(tiling)] * Hh, device=dev)
        nt = L.nt[0]
        qp = torch.empty((1, Hh, L.n_cap, d), dtype=torch.bfloat16, device=dev)
        kp, vp, op = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
        for src, dst in ((q, qp), (k, kp), (v, vp)):
            veda_permute(L, src, dst)
        if o_full is None:        # full attention: the dense path, back in token order
            veda_sparse_attn(L, qp, kp, vp, None, None, 0, scale, op)
            o_full = torch.empty_like(q)
            veda_permute(L, o_full, op, inverse=True)
        # oracle tile map of every query tile of every head; [heads, nt, nt]
        # is the [1, heads, nt_cap, nt_cap] score layout top-k reads
        tm = torch.empty((1, Hh, nt, nt), dtype=torch.float32, device=dev)
        veda_full_attn_tilemax(L, qp, kp, list(range(Hh)), None, nt, scale, tm)
        kk = k_from_keep(keep, nt)
        idx = torch.empty((1, Hh, nt, kk), dtype=torch.int32, device=dev)
        veda_topk_mask(L, tm, [kk] * Hh, kk, idx)
        veda_sparse_attn(L, qp, kp, vp, idx, [kk] * Hh, kk, scale, op)
        o = torch.empty_like(q)
        veda_permute(L, o, op, inverse=True)
        veda_output_sq_error(L, o, o_full, errors[c])
        veda_check_status(L)
    return errors[:, :Hh].cpu()


def choose_tilings(q, k, v, T: int, H: int, W: int, tile: int, candidates: Sequence[Tiling],
                   keep: float, scale: float = None) -> Tuple[List[Tiling], torch.Tensor]:
    """The candidate of smallest error for each head (ties: the earlier
    candidate), and the error table."""
    errors = tiling_errors(q, k, v, T, H, W, tile, candidates, keep, scale)
    best = torch.argmin(errors, dim=0).tolist()
    return [tuple(candidates[i]) for i in best], errors
