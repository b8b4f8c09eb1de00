"""Pins for the fp64 oracle: hand-derived fixtures, closed forms, invariants,
library special cases and brute force on tiny inputs. None of these compare
the oracle with itself; each would fail on a plausible slip (a dropped term, a
wrong sign or index, a transposed operand)."""
import json
import math
import os
from itertools import product

import numpy as np
import pytest
import torch

from oracle import veda_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- permutation

def _perm_by_enumeration(T, H, W, tiling):
    """Independent formulation: walk tiles in (tt, th, tw) order and tokens in
    local (t, y, x) order, emitting the original index or -1."""
    pt, ph, pw = tiling
    out = []
    for tt in range(-(-T // pt)):
        for th in range(H // ph):
            for tw in range(W // pw):
                for lt in range(pt):
                    for ly in range(ph):
                        for lx in range(pw):
                            t, y, x = tt * pt + lt, th * ph + ly, tw * pw + lx
                            out.append((t * H + y) * W + x if t < T else -1)
    return np.array(out)


@pytest.mark.parametrize("name", ["perm_T2H2W4_tiling122.json", "perm_T3H2W2_tiling212_padded.json"])
def test_perm_golden(golden_dir, name):
    g = _load(golden_dir, name)
    perm = O.perm_indices(g["T"], g["H"], g["W"], g["tiling"])
    assert perm.tolist() == g["perm"]
    assert O.head_layout(g["T"], g["H"], g["W"], g["tiling"])["lens"].tolist() == g["lens"]


GRIDS = [(4, 8, 8), (3, 4, 6), (5, 4, 4), (7, 2, 8)]
TILINGS = [(1, 2, 2), (2, 2, 1), (4, 1, 2), (3, 2, 2), (1, 4, 2), (2, 1, 1)]


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("tiling", TILINGS)
def test_perm_matches_enumeration_and_is_bijection(grid, tiling):
    T, H, W = grid
    if H % tiling[1] or W % tiling[2]:
        pytest.skip("tiling does not divide H, W")
    perm = O.perm_indices(T, H, W, tiling)
    assert np.array_equal(perm, _perm_by_enumeration(T, H, W, tiling))
    valid = perm[perm >= 0]
    assert sorted(valid.tolist()) == list(range(T * H * W))
    # valid tokens of every tile are a prefix of the tile
    tile = int(np.prod(tiling))
    lay = O.head_layout(T, H, W, tiling)
    for i, ln in enumerate(lay["lens"]):
        blk = perm[i * tile:(i + 1) * tile]
        assert (blk[:ln] >= 0).all() and (blk[ln:] < 0).all()


def test_perm_identity_tilings():
    T, H, W = 3, 4, 6
    assert np.array_equal(O.perm_indices(T, H, W, (1, H, W)), np.arange(T * H * W))
    assert np.array_equal(O.perm_indices(T, H, W, (T, H, W)), np.arange(T * H * W))


def test_permute_round_trip():
    rng = np.random.default_rng(0)
    T, H, W = 5, 4, 4
    tilings = [(2, 2, 2), (4, 1, 2), (1, 4, 2)]
    perms = [O.perm_indices(T, H, W, t) for t in tilings]
    n_cap = max(len(p) for p in perms)
    x = rng.standard_normal((2, T * H * W, 3, 5))
    xp = O.permute(x, perms, n_cap)
    assert np.array_equal(O.unpermute(xp, perms, T * H * W), x)
    for h, p in enumerate(perms):
        pad = np.nonzero(p < 0)[0]
        assert not xp[:, h, pad].any()
        assert not xp[:, h, len(p):].any()


# ------------------------------------------------------------------- TripPool

def test_trippool_golden(golden_dir):
    g = _load(golden_dir, "trippool_3tokens.json")
    out = O.trippool(np.array(g["rows"], np.float64), np.array([g["len"]]), g["tile"])
    np.testing.assert_allclose(out[0], g["desc"], rtol=0, atol=1e-15)


def test_trippool_invariants_and_brute_force():
    rng = np.random.default_rng(1)
    tile, d = 8, 5
    lens = np.array([8, 3, 1, 8])
    x = rng.standard_normal((len(lens) * tile, d))
    x[tile * 3:] = 2.5                                  # constant tile
    out = O.trippool(x, lens, tile)
    for i, ln in enumerate(lens):
        for c in range(d):
            vals = [x[i * tile + r, c] for r in range(ln)]
            assert out[i, c] == pytest.approx(sum(vals) / ln, abs=1e-14)
            assert out[i, d + c] == max(vals)
            assert out[i, 2 * d + c] == min(vals)
    assert np.all(out[:, 2 * d:] <= out[:, :d] + 1e-15) and np.all(out[:, :d] <= out[:, d:2 * d] + 1e-15)
    np.testing.assert_array_equal(out[3], np.full(3 * d, 2.5))
    np.testing.assert_array_equal(out[2, :d], out[2, d:2 * d])       # single token: avg=max=min


# ------------------------------------------------------------ MLP and scores

def test_gelu_golden(golden_dir):
    g = _load(golden_dir, "gelu_values.json")
    np.testing.assert_allclose(O.gelu(np.array(g["x"])), g["gelu"], rtol=1e-15, atol=1e-16)
    assert O.gelu(np.array([30.0]))[0] == pytest.approx(30.0, rel=1e-15)
    assert abs(O.gelu(np.array([-30.0]))[0]) < 1e-150


def test_mlp_against_loops():
    rng = np.random.default_rng(2)
    din, hid, dout, rows = 6, 4, 3, 5
    x = rng.standard_normal((rows, din))
    w1, b1 = rng.standard_normal((din, hid)), rng.standard_normal(hid)
    w2, b2 = rng.standard_normal((hid, dout)), rng.standard_normal(dout)
    got = O.mlp(x, w1, b1, w2, b2)
    for r in range(rows):
        h = []
        for j in range(hid):
            a = b1[j] + sum(x[r, i] * w1[i, j] for i in range(din))
            h.append(a * 0.5 * (1 + math.erf(a / math.sqrt(2))))
        for o in range(dout):
            want = b2[o] + sum(h[j] * w2[j, o] for j in range(hid))
            assert got[r, o] == pytest.approx(want, rel=1e-12, abs=1e-12)


def test_scores_orientation_and_zero_head():
    rng = np.random.default_rng(3)
    d3, hid, dout = 6, 4, 3
    dq, dk = rng.standard_normal((4, d3)), rng.standard_normal((5, d3))
    w1, b1 = rng.standard_normal((d3, hid)), rng.standard_normal(hid)
    w2, b2 = rng.standard_normal((hid, dout)), rng.standard_normal(dout)
    w1k = rng.standard_normal((d3, hid))
    s = O.tile_scores(dq, dk, w1, b1, w2, b2, w1k, b1, w2, b2, 0.125)
    assert s.shape == (4, 5) and s.dtype == np.float32
    # row i uses query tile i with the q weights, column j key tile j with the k weights
    qi = O.mlp(dq[2:3], w1, b1, w2, b2)[0]
    kj = O.mlp(dk[4:5], w1k, b1, w2, b2)[0]
    assert s[2, 4] == np.float32(float(qi @ kj) * 0.125)
    z = O.tile_scores(dq, dk, w1, b1, np.zeros_like(w2), np.zeros(dout), w1k, b1,
                      np.zeros_like(w2), np.zeros(dout), 0.125)
    assert not z.any()
    idx, _ = O.topk_rows(z, 2)                          # all-equal row: first k tiles
    assert (idx == [0, 1]).all()


# ---------------------------------------------------------------------- top-k

def _brute_force_subsets(row, k):
    nt = len(row)
    out = []
    for bits in product((0, 1), repeat=nt):
        if sum(bits) != k:
            continue
        S = [j for j in range(nt) if bits[j]]
        U = [j for j in range(nt) if not bits[j]]
        if all((row[s] > row[u]) or (row[s] == row[u] and s < u) for s in S for u in U):
            out.append(S)
    return out


def test_topk_golden(golden_dir):
    g = _load(golden_dir, "topk_ties.json")
    row = np.array([g["row"]], np.float32)
    assert O.topk_rows(row, 3)[0][0].tolist() == g["k3"]
    assert O.topk_rows(row, 4)[0][0].tolist() == g["k4"]


def test_topk_brute_force():
    rng = np.random.default_rng(4)
    for trial in range(200):
        nt = int(rng.integers(1, 9))
        k = int(rng.integers(1, nt + 1))
        row = rng.integers(-2, 3, size=nt).astype(np.float32) * np.float32(0.5)   # many ties
        if trial % 3 == 0:
            row = rng.standard_normal(nt).astype(np.float32)
        subs = _brute_force_subsets(row, k)
        assert len(subs) == 1
        idx, mask = O.topk_rows(row[None], k, k_cap=k + 2)
        assert idx[0, :k].tolist() == subs[0] and (idx[0, k:] == -1).all()
        assert mask[0].sum() == k and set(np.nonzero(mask[0])[0]) == set(subs[0])


def test_topk_monotone_rows():
    row = np.arange(10, dtype=np.float32)[None]
    assert O.topk_rows(row, 3)[0][0].tolist() == [7, 8, 9]
    assert O.topk_rows(np.ones((1, 10), np.float32), 3)[0][0].tolist() == [0, 1, 2]


def test_k_from_keep():
    assert O.k_from_keep(0.2, 384) == 77
    assert O.k_from_keep(0.1, 1200) == 120 and O.k_from_keep(0.05, 1200) == 60
    assert O.k_from_keep(0.01, 4) == 1 and O.k_from_keep(1.0, 7) == 7


# ---------------------------------------------------------- sparse attention

def _sdpa_fp64(q, k, v, scale):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], scale=scale)[0, 0].numpy()


def test_attention_two_key_closed_form():
    # one query, two keys with logits 0 and ln 3: weights 1/4, 3/4
    q = np.array([[1.0, 0.0]])
    k = np.array([[0.0, 0.0], [math.log(3.0), 0.0]])
    v = np.array([[4.0, -8.0], [0.0, 4.0]])
    out = O.sparse_attention(q, k, v, np.array([[0]]), 1, np.array([2]), 2, 1.0, rows=[0])
    np.testing.assert_allclose(out[0][0][0], [1.0, 1.0], atol=1e-15)
    assert out[0][1][0] == pytest.approx(math.log(1 + 3.0), abs=1e-15)


@pytest.mark.parametrize("tiling", [(1, 2, 4), (2, 2, 2), (3, 1, 4)])
def test_keep_all_is_full_attention(tiling):
    """Keeping every tile reproduces textbook softmax attention, in original
    token order after unpermute (permutation equivariance)."""
    rng = np.random.default_rng(5)
    T, H, W, d = 5, 2, 4, 8
    tile = int(np.prod(tiling))
    N = T * H * W
    q, k, v = (rng.standard_normal((1, N, 1, d)) for _ in range(3))
    perm = O.perm_indices(T, H, W, tiling)
    lay = O.head_layout(T, H, W, tiling)
    nt, lens = lay["nt"], lay["lens"]
    qp, kp, vp = (O.permute(t, [perm], len(perm))[0, 0] for t in (q, k, v))
    idx = np.tile(np.arange(nt), (nt, 1))
    scale = 1 / math.sqrt(d)
    out = O.sparse_attention(qp, kp, vp, idx, nt, lens, tile, scale)
    op = np.zeros((1, 1, len(perm), d))
    for a, (oa, _) in out.items():
        op[0, 0, a * tile: a * tile + lens[a]] = oa
    got = O.unpermute(op, [perm], N)[0, :, 0]
    want = _sdpa_fp64(q[0, :, 0], k[0, :, 0], v[0, :, 0], scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_brute_force_loops_and_constant_v():
    rng = np.random.default_rng(6)
    tile, d, nt = 4, 3, 4
    lens = np.array([4, 4, 4, 3])
    qp, kp, vp = (rng.standard_normal((nt * tile, d)) for _ in range(3))
    idx = np.array([[1, 3], [0, 2], [2, 3], [0, 1]])
    out = O.sparse_attention(qp, kp, vp, idx, 2, lens, tile, 0.7)
    for a in range(nt):
        keys = [b * tile + j for b in idx[a] for j in range(lens[b])]
        for i in range(lens[a]):
            s = [0.7 * sum(qp[a * tile + i, c] * kp[j, c] for c in range(d)) for j in keys]
            w = [math.exp(x) for x in s]
            z = sum(w)
            for c in range(d):
                want = sum(w[t] * vp[keys[t], c] for t in range(len(keys))) / z
                assert out[a][0][i, c] == pytest.approx(want, rel=1e-12, abs=1e-12)
            assert out[a][1][i] == pytest.approx(math.log(z), rel=1e-12)
    # V constant per tile and k=1: every output row equals that constant
    vc = np.repeat(np.arange(nt, dtype=np.float64) + 0.5, tile)[:, None].repeat(d, axis=1)
    one = O.sparse_attention(qp, kp, vc, idx[:, :1], 1, lens, tile, 0.7)
    for a in range(nt):
        np.testing.assert_allclose(one[a][0], np.full((lens[a], d), idx[a, 0] + 0.5), atol=1e-13)


# -------------------------------------------------------------- tile map, KL

def test_tilemap_brute_force():
    rng = np.random.default_rng(7)
    tile, d, nt = 3, 2, 4
    lens = np.array([3, 3, 2, 3])
    qp, kp = rng.standard_normal((nt * tile, d)), rng.standard_normal((nt * tile, d))
    M, lse = O.full_tilemap(qp, kp, lens, tile, 0.9)
    keys = [(b, b * tile + j) for b in range(nt) for j in range(lens[b])]
    for a in range(nt):
        for b in range(nt):
            best = -1.0
            for i in range(lens[a]):
                logits = [0.9 * sum(qp[a * tile + i, c] * kp[j, c] for c in range(d)) for _, j in keys]
                z = sum(math.exp(x) for x in logits)
                for (bb, _), x in zip(keys, logits):
                    if bb == b:
                        best = max(best, math.exp(x) / z)
                if b == 0:
                    assert lse[a][i] == pytest.approx(math.log(z), rel=1e-12)
            assert M[a, b] == pytest.approx(best, rel=1e-12)
    n_valid = int(lens.sum())
    assert np.all(M.max(axis=1) >= 1.0 / n_valid) and np.all(M <= 1.0)


def test_tilemap_one_hot_gives_expected_mask():
    """Tile-aligned one-hot attention: K rows of tile b = beta*e_b, Q rows of
    tile a = beta*e_sigma(a); the map's top-1 reproduces sigma."""
    tile, d, nt, beta = 4, 8, 6, 16.0
    sigma = [3, 0, 5, 1, 4, 2]
    lens = np.full(nt, tile)
    kp = np.zeros((nt * tile, d))
    qp = np.zeros((nt * tile, d))
    for b in range(nt):
        kp[b * tile:(b + 1) * tile, b] = beta
        qp[b * tile:(b + 1) * tile, sigma[b]] = beta
    M, _ = O.full_tilemap(qp, kp, lens, tile, 1 / math.sqrt(d))
    idx, mask = O.topk_rows(M.astype(np.float32), 1)
    assert idx[:, 0].tolist() == sigma
    np.testing.assert_allclose(M[np.arange(nt), sigma], 1.0 / tile, rtol=1e-12)


def test_kl_golden_and_invariants(golden_dir):
    g = _load(golden_dir, "kl_two_tiles.json")
    for c in g["cases"]:
        got = O.kl_rows(np.array([g["M"]]), np.array([c["scores"]]))[0]
        assert got == pytest.approx(c["kl"], abs=1e-15)
    rng = np.random.default_rng(8)
    M = rng.uniform(0.0, 1.0, (6, 7))
    M[0, 3] = 0.0                                       # 0 log 0 = 0
    s = rng.standard_normal((6, 7))
    kl = O.kl_rows(M, s)
    assert np.all(kl >= -1e-15) and np.isfinite(kl).all()
    Mp = M[1:] + 0.1
    np.testing.assert_allclose(O.kl_rows(Mp, np.log(Mp) + 3.7), 0.0, atol=1e-14)
    # matches the library routine (torch kl_div with log-probability input)
    t = torch.from_numpy(M / M.sum(1, keepdims=True))
    lp = torch.log_softmax(torch.from_numpy(s), dim=1)
    lib = torch.nn.functional.kl_div(lp, t, reduction="none").sum(1).numpy()
    np.testing.assert_allclose(kl, lib, rtol=1e-12, atol=1e-14)


def test_recall_and_effective_pairs():
    M = np.array([[0.1, 0.9, 0.5], [0.7, 0.2, 0.1]])
    _, pred = O.topk_rows(np.array([[0.0, 1.0, 2.0], [2.0, 1.0, 0.0]], np.float32), 2)
    # row 0: pred {1,2} vs ref {1,2}; row 1: pred {0,1} vs ref {0,1}
    assert O.recall(pred, M, 2) == 1.0
    _, pred2 = O.topk_rows(np.array([[2.0, 1.0, 0.0], [2.0, 1.0, 0.0]], np.float32), 2)
    assert O.recall(pred2, M, 2) == pytest.approx(0.75)
    lens = np.array([4, 4, 2])
    idx = np.array([[0, 2], [1, 2], [0, 1]])
    assert O.effective_pairs(lens, idx, 2) == 4 * 6 + 4 * 6 + 2 * 8


# ------------------------------------------------- estimator training (gradients)

_WNAMES = ["w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k"]


def _estimator_problem(seed=0, d3=6, hid=5, od=4, nt=7, nr=3):
    rng = np.random.default_rng(seed)
    W = {"w1q": rng.standard_normal((d3, hid)), "b1q": rng.standard_normal(hid) * 0.1,
         "w2q": rng.standard_normal((hid, od)), "b2q": rng.standard_normal(od) * 0.1,
         "w1k": rng.standard_normal((d3, hid)), "b1k": rng.standard_normal(hid) * 0.1,
         "w2k": rng.standard_normal((hid, od)), "b2k": rng.standard_normal(od) * 0.1}
    dq = rng.standard_normal((nr, d3))
    dk = rng.standard_normal((nt, d3))
    M = rng.uniform(0.01, 1.0, (nr, nt))
    M[0, 2] = 0.0                                   # a zero map entry (0 log 0 = 0)
    return W, dq, dk, M


def test_estimator_grad_finite_differences():
    """Every entry of every weight gradient against a central difference of
    the loss (fp64, step 1e-5): pins each term of the chain rule."""
    W, dq, dk, M = _estimator_problem()
    scale = 0.3
    loss = lambda: O.estimator_loss(dq, dk, *[W[n] for n in _WNAMES], scale, M)
    g = O.estimator_grad(dq, dk, *[W[n] for n in _WNAMES], scale, M)
    for n in _WNAMES:
        a = W[n]
        assert g[n].shape == a.shape
        fd = np.zeros_like(a)
        for i in np.ndindex(a.shape):
            old = a[i]
            a[i] = old + 1e-5
            lp = loss()
            a[i] = old - 1e-5
            lm = loss()
            a[i] = old
            fd[i] = (lp - lm) / 2e-5
        np.testing.assert_allclose(g[n], fd, rtol=0, atol=1e-8 * max(1.0, np.abs(fd).max()), err_msg=n)


def test_estimator_grad_invariants_and_autograd():
    W, dq, dk, M = _estimator_problem(seed=1)
    args = [W[n] for n in _WNAMES]
    g = O.estimator_grad(dq, dk, *args, 0.3, M)
    # a shift of every key embedding adds a per-row constant to the scores:
    # softmax, and so the loss, cannot depend on the key-side output bias
    np.testing.assert_allclose(g["b2k"], 0.0, atol=1e-14)
    # at the minimum (target = the predicted distribution) every gradient is 0
    q = O.mlp(dq, *args[:4])
    k = O.mlp(dk, *args[4:])
    s = q @ k.T * 0.3
    p = np.exp(s - s.max(1, keepdims=True))
    g0 = O.estimator_grad(dq, dk, *args, 0.3, 5.0 * p / p.sum(1, keepdims=True))
    for n in _WNAMES:
        np.testing.assert_allclose(g0[n], 0.0, atol=1e-13)
    # GELU derivative: value at 0, and a difference quotient elsewhere
    assert O.gelu_grad(0.0) == pytest.approx(0.5, abs=1e-15)
    x = np.linspace(-4, 4, 17)
    np.testing.assert_allclose(O.gelu_grad(x), (O.gelu(x + 1e-6) - O.gelu(x - 1e-6)) / 2e-6, atol=1e-8)
    # torch autograd (fp64) on the same loss, built from torch's own ops
    T = {n: torch.tensor(W[n], dtype=torch.float64, requires_grad=True) for n in _WNAMES}
    gel = torch.nn.functional.gelu
    xq, xk = torch.from_numpy(dq), torch.from_numpy(dk)
    qt = gel(xq @ T["w1q"] + T["b1q"]) @ T["w2q"] + T["b2q"]
    kt = gel(xk @ T["w1k"] + T["b1k"]) @ T["w2k"] + T["b2k"]
    lp = torch.log_softmax(qt @ kt.T * 0.3, dim=1)
    tt = torch.from_numpy(M / M.sum(1, keepdims=True))
    torch.nn.functional.kl_div(lp, tt, reduction="none").sum(1).mean().backward()
    for n in _WNAMES:
        np.testing.assert_allclose(g[n], T[n].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)


# ------------------------------------------------------ head-aware tiling search

def test_tiling_errors_keep_all_and_designed_locality():
    """keep = 1 keeps every tile, so every candidate reproduces full attention
    (error 0). With attention confined to each token's own frame (one t), a
    tiling whose tiles are whole frames keeps exactly the right key tile at
    k = 1 (error ~ 0) while tilings that mix frames cannot; head 1 is built
    local in x-columns instead (every frame at one x), which tiles spanning
    all of T (one x column each) capture."""
    T, H, W, d = 4, 2, 4, 8
    N = T * H * W
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    t, y, x = t.ravel(), y.ravel(), x.ravel()
    q = np.zeros((1, N, 2, d))
    k = np.zeros((1, N, 2, d))
    beta = 12.0
    q[0, np.arange(N), 0, t] = beta                 # head 0: one-hot of the frame
    k[0, np.arange(N), 0, t] = beta
    q[0, np.arange(N), 1, x] = beta                 # head 1: one-hot of the x column
    k[0, np.arange(N), 1, x] = beta
    v = np.random.default_rng(3).standard_normal((1, N, 2, d))
    cands = [(1, 2, 4), (4, 2, 1)]                  # whole frames | whole x columns over time
    e_all = O.tiling_errors(q, k, v, T, H, W, cands, 1.0, 1.0)
    np.testing.assert_allclose(e_all, 0.0, atol=1e-20)
    e = O.tiling_errors(q, k, v, T, H, W, cands, 0.25, 1.0)   # k = 1 of 4 tiles
    assert e[0, 0] < 1e-20 and e[1, 0] > 1e-3                # head 0 wants frames
    assert e[1, 1] < 1e-20 and e[0, 1] > 1e-3                # head 1 wants x columns
    assert list(np.argmin(e, axis=0)) == [0, 1]


def test_score_cache_rule_closed_forms():
    """Temporal caching of tile scores (the [reading] of Veda summary 5): the
    refresh rule on cases whose answer is fixed by arithmetic, not by
    re-evaluating the oracle's formula."""
    rng = np.random.default_rng(3)
    B, Hh, nt_cap, din = 1, 3, 6, 12
    nt = [6, 4, 5]
    dq = rng.standard_normal((B, Hh, nt_cap, din))
    dk = rng.standard_normal((B, Hh, nt_cap, din))
    junk = np.full_like(dq, 99.0)
    age = np.full(B * Hh, -1)
    # first step: every head refreshes and takes the descriptors as reference
    r, age, rq, rk = O.score_cache_step(dq, dk, junk, junk, nt, age, tau=0.3, max_age=4)
    assert r.tolist() == [1, 1, 1] and age.tolist() == [0, 0, 0]
    for h in range(Hh):
        assert np.array_equal(rq[0, h, :nt[h]], dq[0, h, :nt[h]])
    # unchanged descriptors: reused while age + 1 < max_age, then refreshed
    seen = []
    for _ in range(4):
        r, age, rq, rk = O.score_cache_step(dq, dk, rq, rk, nt, age, tau=0.3, max_age=4)
        seen.append(r.tolist())
    assert seen == [[0, 0, 0], [0, 0, 0], [0, 0, 0], [1, 1, 1]]
    # scaling Q and K by (1 + eps) moves them by exactly eps relative to the
    # reference: 0.35 > tau refreshes (also when the drift would wrongly be
    # measured against the new descriptors, 0.35/1.35 < 0.3); 0.25 keeps
    age = np.zeros(B * Hh, int)
    r, _, _, _ = O.score_cache_step(dq * 1.35, dk * 1.35, dq, dk, nt, age, tau=0.3, max_age=10)
    assert r.tolist() == [1, 1, 1]
    r, _, _, _ = O.score_cache_step(dq * 1.25, dk * 1.25, dq, dk, nt, age, tau=0.3, max_age=10)
    assert r.tolist() == [0, 0, 0]
    # a change in K alone counts; a change past nt (padding tiles) does not;
    # heads are independent
    dk2 = dk.copy()
    dk2[0, 1, :nt[1]] *= 3.0
    dq3 = dq.copy()
    dq3[0, 2, nt[2]:] += 50.0
    r, age2, rq2, _ = O.score_cache_step(dq3, dk2, dq, dk, nt, age, tau=0.3, max_age=10)
    assert r.tolist() == [0, 1, 0] and age2.tolist() == [1, 0, 1]
    assert np.array_equal(rq2[0, 0], dq[0, 0])
    # max_age = 1 rebuilds every step; tau = 0 rebuilds on any change
    r, _, _, _ = O.score_cache_step(dq, dk, dq, dk, nt, age, tau=0.3, max_age=1)
    assert r.tolist() == [1, 1, 1]
    dq4 = dq.copy()
    dq4[0, 0, 0, 0] += 1e-9
    r, _, _, _ = O.score_cache_step(dq4, dk, dq, dk, nt, age, tau=0.0, max_age=10)
    assert r.tolist() == [1, 0, 0]
