"""Plain fp64 CPU oracle for the Veda tile-selection front end and the
tile-skipping sparse attention layer.

TEST INFRASTRUCTURE ONLY. This module is the independent reference that the
CUDA library is checked against. Only the test suite, the package's smoke
check and the benchmark's CPU-baseline leg may import it; the library never
does. It shares no code, table or helper with the CUDA path and imports
nothing but NumPy and the standard library.

Source: "Technical Summary: Veda - Scalable Video Diffusion via Distilled
Sparse Attention" (gist.science, arXiv 2605.30325), cited below as "Veda
summary", with its section numbers. The pages describe the method in named
steps only; every point they leave open follows the plainest reading, marked
[reading] and listed in the design notes.

Conventions
  * Q, K, V arrive as [B, N, heads, d] arrays holding bf16 values (upcast to
    float64 here); original token order n = (t*H + y)*W + x   [reading].
  * A tiling pi = (p_t, p_h, p_w) with p_t*p_h*p_w == tile   (Veda summary 2.2).
  * Every accumulation is float64; fp32 is used only where the result is an
    fp32 quantity by definition (the emitted tile scores that top-k ranks).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "head_layout", "perm_indices", "permute", "unpermute", "trippool", "gelu",
    "mlp", "tile_scores", "topk_rows", "sparse_attention", "full_tilemap",
    "kl_rows", "recall", "k_from_keep", "effective_pairs",
    "gelu_grad", "estimator_loss", "estimator_grad", "tiling_errors",
    "score_cache_step",
]


# ---------------------------------------------------------------------------
# 1. head-aware tiling permutation (Veda summary 2.2, "Head-Aware Tiling")
# ---------------------------------------------------------------------------

def head_layout(T, H, W, tiling):
    """Tile counts of one head's tiling.

    [reading] H and W are divisible by p_h and p_w; T is padded at its end to
    a multiple of p_t. Tiles are numbered row-major over (tile_t, tile_h,
    tile_w); tokens inside a tile row-major over local (t, y, x), so the
    valid tokens of every tile form a prefix of the tile.

    Returns dict(nt, n_pad, lens) with lens[i] = valid tokens of tile i.
    """
    pt, ph, pw = (int(v) for v in tiling)
    if H % ph or W % pw:
        raise ValueError("p_h and p_w must divide H and W")
    ntt = -(-T // pt)
    nht, nwt = H // ph, W // pw
    nt = ntt * nht * nwt
    tile = pt * ph * pw
    lens = np.empty(nt, np.int64)
    for i in range(nt):
        tt = i // (nht * nwt)
        lens[i] = min(pt, T - tt * pt) * ph * pw
    return {"nt": nt, "n_pad": nt * tile, "lens": lens, "tile": tile}


def perm_indices(T, H, W, tiling):
    """perm[slot] = original token index, or -1 for a padding slot.

    slot = tile_id*tile + local, tile_id = ((t//p_t)*nH + y//p_h)*nW + x//p_w,
    local = ((t%p_t)*p_h + y%p_h)*p_w + x%p_w.
    """
    pt, ph, pw = (int(v) for v in tiling)
    lay = head_layout(T, H, W, tiling)
    tile = lay["tile"]
    nht, nwt = H // ph, W // pw
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    n = (t * H + y) * W + x
    tid = ((t // pt) * nht + y // ph) * nwt + x // pw
    loc = ((t % pt) * ph + y % ph) * pw + x % pw
    perm = np.full(lay["n_pad"], -1, np.int64)
    perm[(tid * tile + loc).ravel()] = n.ravel()
    return perm


def permute(x, perms, n_cap):
    """[B, N, heads, d] -> [B, heads, n_cap, d]; padding slots are zero."""
    B, N, Hh, d = x.shape
    out = np.zeros((B, Hh, n_cap, d), dtype=np.float64)
    for h in range(Hh):
        p = perms[h]
        valid = p >= 0
        slots = np.nonzero(valid)[0]
        out[:, h, slots, :] = x[:, p[valid], h, :]
    return out


def unpermute(xp, perms, N):
    """Inverse of ``permute``: [B, heads, n_cap, d] -> [B, N, heads, d]; rows
    of padding slots are dropped."""
    B, Hh, n_cap, d = xp.shape
    out = np.zeros((B, N, Hh, d), dtype=np.float64)
    for h in range(Hh):
        p = perms[h]
        valid = p >= 0
        out[:, p[valid], h, :] = xp[:, h, np.nonzero(valid)[0], :]
    return out


# ---------------------------------------------------------------------------
# 2. TripPool descriptor (Veda summary 2.1, "Statistic-Aware Estimator")
# ---------------------------------------------------------------------------

def trippool(xp_head, lens, tile):
    """Per tile, per channel: [mean | max | min] over the tile's valid tokens.

    xp_head: [n_slots, d] permuted rows of one head. Returns [nt, 3d]."""
    nt = len(lens)
    d = xp_head.shape[1]
    out = np.empty((nt, 3 * d), np.float64)
    for i in range(nt):
        rows = xp_head[i * tile: i * tile + int(lens[i])]
        out[i, :d] = rows.mean(axis=0)
        out[i, d:2 * d] = rows.max(axis=0)
        out[i, 2 * d:] = rows.min(axis=0)
    return out


# ---------------------------------------------------------------------------
# 3. head-specific MLP estimator and tile scores (Veda summary 2.1,
#    "Head-Specific Projections")
# ---------------------------------------------------------------------------

def gelu(x):
    """Exact GELU, x * Phi(x) with Phi the standard normal CDF (erf form)."""
    x = np.asarray(x, np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def mlp(desc, w1, b1, w2, b2):
    """One head's estimator: Linear(3d, hidden) -> GELU -> Linear(hidden, out).
    Weight layout [in, out] (row vector times matrix)."""
    h = desc @ np.asarray(w1, np.float64) + np.asarray(b1, np.float64)
    return gelu(h) @ np.asarray(w2, np.float64) + np.asarray(b2, np.float64)


def tile_scores(dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale):
    """Predicted tile-level scores of one head: score[i, j] = q_i . k_j * scale,
    q = MLP_q(TripPool(Q tile i)), k = MLP_k(TripPool(K tile j)). Computed in
    fp64 and returned as float32, the precision the top-k step ranks in."""
    q = mlp(dq, w1q, b1q, w2q, b2q)
    k = mlp(dk, w1k, b1k, w2k, b2k)
    return (q @ k.T * scale).astype(np.float32)


# ---------------------------------------------------------------------------
# 4. top-k key tiles per query tile (Veda summary 2.1 and section 4: only the
#    highest-scoring tiles are kept, 90-95% of them skipped)
# ---------------------------------------------------------------------------

def k_from_keep(keep, nt):
    """[reading] kept key tiles per row: round-half-up of keep*nt, at least 1."""
    return max(1, int(math.floor(keep * nt + 0.5)))


def topk_rows(scores, k, k_cap=None):
    """For each row of float32 scores [rows, nt]: the k largest, exact ties
    broken toward the lower tile index (-0.0 ties +0.0). Returns (idx, mask):
    idx [rows, k_cap] int32 ascending, -1 padded; mask [rows, nt] uint8."""
    s = np.asarray(scores, np.float32)
    rows, nt = s.shape
    k_cap = k if k_cap is None else k_cap
    idx = np.full((rows, k_cap), -1, np.int32)
    mask = np.zeros((rows, nt), np.uint8)
    cols = np.arange(nt)
    for r in range(rows):
        # primary key: value descending; secondary: tile index ascending
        order = np.lexsort((cols, -s[r]))
        sel = np.sort(order[:k])
        idx[r, :k] = sel
        mask[r, sel] = 1
    return idx, mask


# ---------------------------------------------------------------------------
# 5. tile-skipping sparse attention (Veda summary 2.3): softmax over the keys
#    of the kept tiles only; skipped tiles contribute nothing.
# ---------------------------------------------------------------------------

def _tile_rows(lens, tile, tiles):
    return np.concatenate([np.arange(b * tile, b * tile + int(lens[b])) for b in tiles])


def sparse_attention(qp_h, kp_h, vp_h, idx_h, k, lens, tile, scale, rows=None):
    """One head. qp_h/kp_h/vp_h: [n_slots, d] permuted rows; idx_h [nt, >=k].
    Returns {a: (O_a [len_a, d], lse_a [len_a])} for each query tile a in
    ``rows`` (default all): O_i = sum_j softmax_j(q_i.k_j*scale) v_j over the
    valid keys j of tiles idx_h[a, :k]."""
    nt = len(lens)
    rows = range(nt) if rows is None else rows
    out = {}
    for a in rows:
        qi = qp_h[a * tile: a * tile + int(lens[a])]
        keys = _tile_rows(lens, tile, [int(b) for b in idx_h[a, :k]])
        s = (qi @ kp_h[keys].T) * scale
        m = s.max(axis=1, keepdims=True)
        w = np.exp(s - m)
        z = w.sum(axis=1, keepdims=True)
        out[a] = ((w @ vp_h[keys]) / z, (m + np.log(z))[:, 0])
    return out


# ---------------------------------------------------------------------------
# 6. oracle tile map: max-pool of the full softmax attention matrix over
#    query-key tile regions (Veda summary 2.1, "Target Construction"; the
#    heat map is produced in two passes, 2.3 "Training Efficiency")
# ---------------------------------------------------------------------------

def full_tilemap(qp_h, kp_h, lens, tile, scale, rows=None):
    """One head. Returns (M [len(rows), nt], lse {a: [len_a]}) with
    M[r, b] = max over valid rows i of query tile rows[r] and valid keys j of
    key tile b of P_ij, P = softmax over all valid keys of the head."""
    nt = len(lens)
    rows = list(range(nt)) if rows is None else list(rows)
    keys = _tile_rows(lens, tile, range(nt))
    col_tile = np.concatenate([np.full(int(lens[b]), b) for b in range(nt)])
    M = np.zeros((len(rows), nt), np.float64)
    lse = {}
    for r, a in enumerate(rows):
        qi = qp_h[a * tile: a * tile + int(lens[a])]
        s = (qi @ kp_h[keys].T) * scale
        m = s.max(axis=1, keepdims=True)
        w = np.exp(s - m)
        z = w.sum(axis=1, keepdims=True)
        P = w / z
        lse[a] = (m + np.log(z))[:, 0]
        colmax = P.max(axis=0)
        M[r] = np.full(nt, -np.inf)
        np.maximum.at(M[r], col_tile, colmax)
    return M, lse


# ---------------------------------------------------------------------------
# 7. row-wise KL distillation loss (Veda summary 2.1, "Optimization") and
#    recall of the predicted mask against the oracle map
# ---------------------------------------------------------------------------

def kl_rows(M_rows, score_rows):
    """[reading] KL(t || p) per row, t = tile-map row normalised to sum 1,
    p = softmax of the predicted score row; 0*log 0 = 0."""
    M = np.asarray(M_rows, np.float64)
    s = np.asarray(score_rows, np.float64)
    t = M / M.sum(axis=1, keepdims=True)
    m = s.max(axis=1, keepdims=True)
    logp = s - m - np.log(np.exp(s - m).sum(axis=1, keepdims=True))
    with np.errstate(divide="ignore", invalid="ignore"):
        terms = np.where(t > 0, t * (np.log(t) - logp), 0.0)
    return terms.sum(axis=1)


def recall(pred_mask_rows, M_rows, k):
    """Mean over rows of |topk(pred) & topk(M)| / k (same tie rule)."""
    _, ref = topk_rows(np.asarray(M_rows, np.float32), k)
    pred = np.asarray(pred_mask_rows, bool)
    return float((pred & ref.astype(bool)).sum(axis=1).mean() / k)


def effective_pairs(lens, idx_h, k, rows=None):
    """Kept valid (query, key) token pairs of one head: the work unit of the
    effective-FLOP count 4*d*pairs."""
    nt = len(lens)
    rows = range(nt) if rows is None else rows
    kl = np.asarray(lens, np.int64)
    return int(sum(int(kl[a]) * int(kl[np.asarray(idx_h[a, :k])].sum()) for a in rows))



# ---------------------------------------------------------------------------
# 8. estimator training (Veda summary 2.1, "Optimization": the head-specific
#    projections are trained with a row-wise KL against the oracle tile map,
#    with stop-gradient on the pooled descriptors; 2.3, "Training Efficiency":
#    on random subsets of query tiles)
# ---------------------------------------------------------------------------

def gelu_grad(x):
    """d/dx of the exact GELU: Phi(x) + x * phi(x), phi the standard normal
    density."""
    x = np.asarray(x, np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * (1.0 + erf(x / math.sqrt(2.0))) + x * np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def estimator_loss(dq_rows, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale, M_rows):
    """[reading] One head's distillation loss: the mean over the sampled query
    tiles (rows of dq_rows, with their tile-map rows M_rows) of KL(t || p),
    t = map row / its sum, p = softmax of the predicted score row over all of
    the head's key tiles (dk). Scores stay fp64 here (no fp32 rounding), so
    the loss is a smooth function of the weights."""
    q = mlp(dq_rows, w1q, b1q, w2q, b2q)
    k = mlp(dk, w1k, b1k, w2k, b2k)
    return float(kl_rows(M_rows, q @ k.T * scale).mean())


def estimator_grad(dq_rows, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scale, M_rows):
    """Gradient of estimator_loss with respect to the eight weight arrays,
    returned as a dict {"w1q", "b1q", "w2q", "b2q", "w1k", ...} in the
    weights' own shapes; descriptors and the tile map are constants.

    Chain rule, written out: with G = (p - t) / rows the gradient of the loss
    with respect to the score matrix (KL(t || softmax(s)) has gradient p - t
    in s because t sums to 1), the score s = scale * q k^T gives
    dq = scale G k and dk = scale G^T q; each side's MLP y = GELU(x W1 + b1)
    W2 + b2 then gives dW2 = GELU(z)^T dy, db2 = sum dy, dz = (dy W2^T) *
    GELU'(z), dW1 = x^T dz, db1 = sum dz."""
    f = lambda a: np.asarray(a, np.float64)
    xq, xk = f(dq_rows), f(dk)
    zq = xq @ f(w1q) + f(b1q)
    zk = xk @ f(w1k) + f(b1k)
    hq, hk = gelu(zq), gelu(zk)
    q = hq @ f(w2q) + f(b2q)
    k = hk @ f(w2k) + f(b2k)
    s = q @ k.T * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    M = f(M_rows)
    t = M / M.sum(axis=1, keepdims=True)
    G = (p - t) / s.shape[0]
    dy = {"q": scale * G @ k, "k": scale * G.T @ q}
    out = {}
    for side, x, z, h, w2 in (("q", xq, zq, hq, f(w2q)), ("k", xk, zk, hk, f(w2k))):
        g = dy[side]
        dz = (g @ w2.T) * gelu_grad(z)
        out["w1" + side] = x.T @ dz
        out["b1" + side] = dz.sum(axis=0)
        out["w2" + side] = h.T @ g
        out["b2" + side] = g.sum(axis=0)
    return out


# ---------------------------------------------------------------------------
# 9. head-aware tiling search (Veda summary 2.2: a tiling per head, chosen
#    offline on calibration inputs to match that head's locality)
# ---------------------------------------------------------------------------

def tiling_errors(q, k, v, T, H, W, candidates, keep, scale):
    """[reading] Calibration score of each candidate tiling for each head:
    squared Frobenius distance, over the head's tokens, between full attention
    and the tile-skipping attention that keeps, for every query tile, the k
    key tiles with the largest oracle tile-map values (the mask the estimator
    is distilled towards), all under that tiling. The chosen tiling of head h
    is argmin over candidates of errors[c, h].

    q, k, v: [1, N, heads, d] (bf16 values). Returns errors [len(candidates),
    heads] (fp64)."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    B, N, Hh, d = q.shape
    assert B == 1
    # full attention in the original order, per head (tiling-independent)
    full = np.zeros((N, Hh, d))
    for h in range(Hh):
        s = q[0, :, h] @ k[0, :, h].T * scale
        w = np.exp(s - s.max(axis=1, keepdims=True))
        full[:, h] = (w / w.sum(axis=1, keepdims=True)) @ v[0, :, h]
    errors = np.zeros((len(candidates), Hh))
    for c, tiling in enumerate(candidates):
        lay = head_layout(T, H, W, tiling)
        perm = perm_indices(T, H, W, tiling)
        perms = [perm] * Hh
        nt, lens, tile = lay["nt"], lay["lens"], lay["tile"]
        kk = k_from_keep(keep, nt)
        qp, kp, vp = (permute(a, perms, lay["n_pad"]) for a in (q, k, v))
        op = np.zeros((1, Hh, lay["n_pad"], d))
        for h in range(Hh):
            M, _ = full_tilemap(qp[0, h], kp[0, h], lens, tile, scale)
            idx, _ = topk_rows(M.astype(np.float32), kk)
            for a, (oa, _) in sparse_attention(qp[0, h], kp[0, h], vp[0, h], idx, kk, lens, tile, scale).items():
                op[0, h, a * tile: a * tile + int(lens[a])] = oa
        o = unpermute(op, perms, N)[0]
        errors[c] = ((o - full) ** 2).sum(axis=(0, 2))
    return errors


# ---------------------------------------------------------------------------
# 10. temporal caching of tile scores across diffusion steps (Veda summary 5
#     names "temporal caching of tile scores" and adaptive sparsity across
#     timesteps as future work; the rule is a [reading]: a head keeps the
#     mask of its last refresh while its TripPool descriptors stay within a
#     relative distance tau of that step's, for fewer than max_age steps)
# ---------------------------------------------------------------------------

def score_cache_step(dq, dk, dq_ref, dk_ref, nt, age, tau, max_age):
    """One step of the cache rule for every (batch element, head).

    dq, dk, dq_ref, dk_ref: [B, heads, nt_cap, 3d]; nt: tiles per head; age:
    int array [B*heads], -1 = never scored. drift^2 = (|dq - dq_ref|^2 +
    |dk - dk_ref|^2) / (|dq_ref|^2 + |dk_ref|^2) over the head's nt valid
    tiles. Refresh when never scored, when age + 1 >= max_age, or when
    drift^2 > tau^2 (compared as drift^2 numerator <= tau^2 * denominator).
    Returns (refresh [B*heads] int, new age, new dq_ref, new dk_ref)."""
    dq, dk = np.asarray(dq, np.float64), np.asarray(dk, np.float64)
    dq_ref, dk_ref = np.array(dq_ref, np.float64), np.array(dk_ref, np.float64)
    B, Hh = dq.shape[:2]
    age = np.asarray(age, np.int64).copy()
    refresh = np.zeros(B * Hh, np.int64)
    for b in range(B):
        for h in range(Hh):
            i, n = b * Hh + h, int(nt[h])
            num = ((dq[b, h, :n] - dq_ref[b, h, :n]) ** 2).sum() + ((dk[b, h, :n] - dk_ref[b, h, :n]) ** 2).sum()
            den = (dq_ref[b, h, :n] ** 2).sum() + (dk_ref[b, h, :n] ** 2).sum()
            fresh = age[i] < 0 or age[i] + 1 >= max_age or not (num <= tau * tau * den)
            refresh[i] = int(fresh)
            if fresh:
                age[i] = 0
                dq_ref[b, h, :n], dk_ref[b, h, :n] = dq[b, h, :n], dk[b, h, :n]
            else:
                age[i] += 1
    return refresh, age, dq_ref, dk_ref
