"""Planted mistakes: each case swaps one oracle function for a copy with a
plausible slip and checks that at least one pin in test_oracle.py fails. This
shows the pins discriminate; the oracle itself is never modified on disk."""
import inspect
import math

import numpy as np
import pytest

from oracle import veda_oracle as O
from tests import test_oracle as P

_orig = {name: getattr(O, name) for name in O.__all__}


def _perm_x_major(T, H, W, tiling):
    """slip: tokens inside a tile ordered x-major instead of t-major."""
    pt, ph, pw = tiling
    perm = _orig["perm_indices"](T, H, W, tiling)
    tile = pt * ph * pw
    out = perm.copy()
    for b in range(len(perm) // tile):
        blk = perm[b * tile:(b + 1) * tile].reshape(pt, ph, pw)
        out[b * tile:(b + 1) * tile] = blk.transpose(2, 1, 0).ravel()
    return out


def _trippool_no_max(xp_head, lens, tile):
    """slip: dropped max term (mean repeated)."""
    out = _orig["trippool"](xp_head, lens, tile)
    d = xp_head.shape[1]
    out[:, d:2 * d] = out[:, :d]
    return out


def _scores_transposed(dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale):
    """slip: query and key weights swapped."""
    return _orig["tile_scores"](dq, dk, w1k, b1k, w2k, b2k, w1q, b1q, w2q, b2q, scale)


def _topk_high_ties(scores, k, k_cap=None):
    """slip: exact ties broken toward the higher index."""
    s = np.asarray(scores, np.float32)
    flipped = s[:, ::-1]
    idx, mask = _orig["topk_rows"](flipped, k, k_cap)
    nt = s.shape[1]
    idx = np.where(idx >= 0, nt - 1 - idx, -1)
    idx[:, :k] = np.sort(idx[:, :k], axis=1)
    return idx, mask[:, ::-1].copy()


def _attn_double_scale(qp_h, kp_h, vp_h, idx_h, k, lens, tile, scale, rows=None):
    """slip: scale applied twice."""
    return _orig["sparse_attention"](qp_h, kp_h, vp_h, idx_h, k, lens, tile, scale * scale, rows)


def _attn_no_renorm(qp_h, kp_h, vp_h, idx_h, k, lens, tile, scale, rows=None):
    """slip: softmax normaliser taken over every key, not only the kept ones."""
    nt = len(lens)
    full = _orig["sparse_attention"](qp_h, kp_h, vp_h, np.tile(np.arange(nt), (nt, 1)), nt, lens, tile, scale, rows)
    part = _orig["sparse_attention"](qp_h, kp_h, vp_h, idx_h, k, lens, tile, scale, rows)
    return {a: (part[a][0] * np.exp(part[a][1] - full[a][1])[:, None], full[a][1]) for a in part}


def _tilemap_mean(qp_h, kp_h, lens, tile, scale, rows=None):
    """slip: average-pooling of the attention matrix instead of max-pooling."""
    M, lse = _orig["full_tilemap"](qp_h, kp_h, lens, tile, scale, rows)
    nt = len(lens)
    rows = list(range(nt)) if rows is None else list(rows)
    out = np.zeros_like(M)
    keys = np.concatenate([np.arange(b * tile, b * tile + int(lens[b])) for b in range(nt)])
    col_tile = np.concatenate([np.full(int(lens[b]), b) for b in range(nt)])
    for r, a in enumerate(rows):
        qi = qp_h[a * tile: a * tile + int(lens[a])]
        s = (qi @ kp_h[keys].T) * scale
        P_ = np.exp(s - lse[a][:, None])
        for b in range(nt):
            out[r, b] = P_[:, col_tile == b].mean()
    return out, lse


def _kl_reversed(M_rows, score_rows):
    """slip: KL direction reversed, KL(p || t)."""
    M = np.asarray(M_rows, np.float64)
    s = np.asarray(score_rows, np.float64)
    t = M / M.sum(axis=1, keepdims=True)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(p > 0, p * (np.log(p) - np.log(t)), 0.0).sum(axis=1)


def _gelu_tanh(x):
    """slip: tanh approximation instead of the exact erf GELU."""
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _grad_no_row_mean(dq_rows, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale, M_rows):
    """slip: gradient of the row sum instead of the row mean."""
    g = _orig["estimator_grad"](dq_rows, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale, M_rows)
    return {n: v * np.asarray(dq_rows).shape[0] for n, v in g.items()}


def _gelu_grad_as_gelu(x):
    """slip: GELU itself used where its derivative belongs."""
    return _orig["gelu"](x)


def _grad_sign_flipped(dq_rows, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale, M_rows):
    """slip: t - p instead of p - t (ascent direction)."""
    g = _orig["estimator_grad"](dq_rows, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale, M_rows)
    return {n: -v for n, v in g.items()}


def _tiling_errors_sparsity_for_keep(q, k, v, T, H, W, candidates, keep, scale):
    """slip: the sparsity (1 - keep) used where the keep fraction belongs."""
    return _orig["tiling_errors"](q, k, v, T, H, W, candidates, 1.0 - keep, scale)


CASES = [
    ("perm_indices", _perm_x_major, ["test_perm_golden"]),
    ("trippool", _trippool_no_max, ["test_trippool_golden", "test_trippool_invariants_and_brute_force"]),
    ("tile_scores", _scores_transposed, ["test_scores_orientation_and_zero_head"]),
    ("topk_rows", _topk_high_ties, ["test_topk_golden", "test_topk_brute_force"]),
    ("sparse_attention", _attn_double_scale, ["test_attention_brute_force_loops_and_constant_v", "test_keep_all_is_full_attention"]),
    ("sparse_attention", _attn_no_renorm, ["test_attention_brute_force_loops_and_constant_v"]),
    ("full_tilemap", _tilemap_mean, ["test_tilemap_brute_force", "test_tilemap_one_hot_gives_expected_mask"]),
    ("kl_rows", _kl_reversed, ["test_kl_golden_and_invariants"]),
    ("gelu", _gelu_tanh, ["test_gelu_golden", "test_mlp_against_loops"]),
    ("estimator_grad", _grad_no_row_mean, ["test_estimator_grad_finite_differences"]),
    ("gelu_grad", _gelu_grad_as_gelu, ["test_estimator_grad_finite_differences"]),
    ("estimator_grad", _grad_sign_flipped, ["test_estimator_grad_finite_differences",
                                            "test_estimator_grad_invariants_and_autograd"]),
    ("tiling_errors", _tiling_errors_sparsity_for_keep, ["test_tiling_errors_keep_all_and_designed_locality"]),
]


def _run_pin(name, golden_dir):
    fn = getattr(P, name)
    params = inspect.signature(fn).parameters
    if "golden_dir" in params and "name" in params:
        for n in ("perm_T2H2W4_tiling122.json", "perm_T3H2W2_tiling212_padded.json"):
            fn(golden_dir, n)
    elif "golden_dir" in params:
        fn(golden_dir)
    elif "tiling" in params:
        fn((2, 2, 2))
    else:
        fn()


@pytest.mark.parametrize("target,mutant,pins", CASES, ids=[c[1].__name__ for c in CASES])
def test_pins_catch_planted_mistake(monkeypatch, golden_dir, target, mutant, pins):
    monkeypatch.setattr(O, target, mutant)
    caught = 0
    for name in pins:
        try:
            _run_pin(name, golden_dir)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught {mutant.__name__}"
