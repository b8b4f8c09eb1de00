"""Test-side glue: builds device inputs from the seeded workloads and the
oracle's view of the same layer. Holds no arithmetic of the method."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import veda_oracle as O


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def oracle_geometry(w: synth.Workload):
    lays = [O.head_layout(w.T, w.H, w.W, t) for t in w.tilings]
    perms = [O.perm_indices(w.T, w.H, w.W, t) for t in w.tilings]
    n_cap = max(l["n_pad"] for l in lays)
    nt_cap = max(l["nt"] for l in lays)
    return lays, perms, n_cap, nt_cap


def oracle_k(w: synth.Workload, lays):
    if w.k_fixed is not None:
        return [min(w.k_fixed, l["nt"]) for l in lays]
    return [O.k_from_keep(w.keep, l["nt"]) for l in lays]


def small_workloads():
    """Small layers that still span several tiles and ragged tails."""
    return {
        "cfg0": synth.config(0),
        "ragged-d128-t128": synth.custom("ragged", 1, 4, 128, 5, 8, 16, 128,
                                         [(2, 8, 8), (4, 4, 8), (1, 8, 16), (8, 4, 4)], 0.4, 21),
        "odd-d128-t64": synth.custom("odd", 1, 3, 128, 3, 8, 8, 64, [(1, 8, 8), (2, 4, 8), (4, 4, 4)], 0.5, 22),
        "batch2-d64-t128": synth.custom("b2", 2, 2, 64, 4, 8, 8, 128, [(2, 8, 8), (4, 4, 8)], 0.5, 23),
        "d64-t64-padded": synth.custom("p64", 1, 2, 64, 7, 4, 8, 64, [(2, 4, 8), (4, 2, 8)], 0.3, 24),
        "single-tile": synth.custom("one", 1, 2, 128, 1, 8, 16, 128, [(1, 8, 16), (1, 8, 16)], 1.0, 25),
    }
