"""GPU parity: every libveda kernel against the fp64 oracle on the same seeded
inputs, each stage fed the same upstream values as the oracle (top-k gets
the oracle's fp32 scores, attention gets the oracle's index lists).

Tolerances (from the method's precision):
  permutation, top-k indices and mask: bit-exact;
  TripPool: max/min exact, mean within 1e-6 relative (fp32 sum of bf16);
  tile scores, tile map, KL: per row max|gpu-oracle| <= 1e-3 * max|oracle|;
  attention output (bf16 in, bf16 out): max abs <= 2e-2, mean abs <= 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_24_b200 as V
import synth
from oracle import veda_oracle as O
from tests.helpers import f64, oracle_geometry, oracle_k, small_workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"
WL = small_workloads()


def _layer(w):
    return V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device=DEV)


def _inputs(w):
    return [t.to(DEV) for t in synth.qkv(w, "cpu")]


def _permuted(L, w, x):
    xp = torch.empty((w.B, w.heads, L.n_cap, w.d), dtype=torch.bfloat16, device=DEV)
    perm = torch.empty((w.heads, L.n_cap), dtype=torch.int32, device=DEV)
    V.veda_permute(L, x, xp, perm)
    return xp, perm


def _check_attention(out, lse, ref, lens, tile, tol_max=2e-2, tol_mean=2e-3):
    errs = []
    for a, (oa, la) in ref.items():
        got = out[a * tile: a * tile + lens[a]]
        errs.append(np.abs(got - oa))
        np.testing.assert_allclose(lse[a * tile: a * tile + lens[a]], la, rtol=1e-3, atol=1e-3)
    e = np.concatenate([x.ravel() for x in errs])
    assert e.max() <= tol_max, e.max()
    assert e.mean() <= tol_mean, e.mean()


def _row_rel(got, want, tol=1e-3, floor=1e-30):
    for g, w_ in zip(np.atleast_2d(got), np.atleast_2d(want)):
        scale = max(np.abs(w_).max(), floor)
        assert np.abs(g - w_).max() <= tol * scale, (np.abs(g - w_).max(), scale)


# ------------------------------------------------------------- permutation

@pytest.mark.parametrize("name", list(WL))
def test_permute_bit_exact_and_round_trip(name):
    w = WL[name]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    assert (L.n_cap, L.nt_cap) == (n_cap, nt_cap)
    q, k, v = _inputs(w)
    qp, perm = _permuted(L, w, q)
    pg = perm.cpu().numpy()
    for h in range(w.heads):
        assert np.array_equal(pg[h, :len(perms[h])], perms[h])
        assert (pg[h, len(perms[h]):] == -1).all()
    want = O.permute(f64(q), perms, n_cap)
    assert np.array_equal(f64(qp), want)
    back = torch.empty_like(q)
    V.veda_permute(L, back, qp, inverse=True)
    torch.cuda.synchronize()
    assert torch.equal(back, q)
    V.veda_check_status(L)


# ---------------------------------------------------------------- TripPool

@pytest.mark.parametrize("name", list(WL))
def test_trippool(name):
    w = WL[name]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, _, _ = _inputs(w)
    qp, _ = _permuted(L, w, q)
    desc = torch.empty((w.B, w.heads, nt_cap, 3 * w.d), dtype=torch.float32, device=DEV)
    V.veda_trippool(L, qp, desc)
    got = desc.cpu().double().numpy()
    xp = f64(qp)
    d = w.d
    for b in range(w.B):
        for h in range(w.heads):
            ref = O.trippool(xp[b, h], lays[h]["lens"], w.tile)
            nt = lays[h]["nt"]
            np.testing.assert_allclose(got[b, h, :nt, :d], ref[:, :d], rtol=1e-6, atol=1e-6)
            assert np.array_equal(got[b, h, :nt, d:], ref[:, d:])
            assert not got[b, h, nt:].any()


@pytest.mark.parametrize("name", list(WL))
def test_permute_trippool_fused(name):
    """The fused call against the oracle (permutation and max/min bit-exact,
    mean within fp32 rounding) and against the two unfused calls."""
    w = WL[name]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, _, _ = _inputs(w)
    xp = torch.full((w.B, w.heads, n_cap, w.d), 7.0, dtype=torch.bfloat16, device=DEV)   # poisoned
    perm = torch.full((w.heads, n_cap), 12345, dtype=torch.int32, device=DEV)
    desc = torch.full((w.B, w.heads, nt_cap, 3 * w.d), 7.0, dtype=torch.float32, device=DEV)
    V.veda_permute_trippool(L, q, xp, desc, perm)
    V.veda_check_status(L)
    pg = perm.cpu().numpy()
    for h in range(w.heads):
        assert np.array_equal(pg[h, :len(perms[h])], perms[h])
        assert (pg[h, len(perms[h]):] == -1).all()
    assert np.array_equal(f64(xp), O.permute(f64(q), perms, n_cap))
    got, d = desc.cpu().double().numpy(), w.d
    for b in range(w.B):
        for h in range(w.heads):
            nt = lays[h]["nt"]
            ref = O.trippool(f64(xp)[b, h], lays[h]["lens"], w.tile)
            np.testing.assert_allclose(got[b, h, :nt, :d], ref[:, :d], rtol=1e-6, atol=1e-6)
            assert np.array_equal(got[b, h, :nt, d:], ref[:, d:])
            assert not got[b, h, nt:].any()
    # same max/min as the unfused TripPool; the permuted tensor identical
    xp2, _ = _permuted(L, w, q)
    desc2 = torch.empty_like(desc)
    V.veda_trippool(L, xp2, desc2)
    torch.cuda.synchronize()
    assert torch.equal(xp, xp2)
    assert torch.equal(desc[..., d:], desc2[..., d:])
    # no perm map requested
    V.veda_permute_trippool(L, q, xp, desc)
    V.veda_check_status(L)


# ------------------------------------------------------------- tile scores

@pytest.mark.parametrize("name", list(WL))
def test_tile_scores(name):
    w = WL[name]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    rng = np.random.default_rng(5)
    dq = rng.standard_normal((w.B, w.heads, nt_cap, 3 * w.d)).astype(np.float32)
    dk = rng.standard_normal((w.B, w.heads, nt_cap, 3 * w.d)).astype(np.float32)
    w1, b1, w2, b2 = synth.mlp_weights(w)
    b1 = rng.standard_normal(b1.shape).astype(np.float32) * 0.1   # exercise the biases
    b2 = rng.standard_normal(b2.shape).astype(np.float32) * 0.1
    w1k = synth.mlp_weights(synth.custom("k", 1, w.heads, w.d, 1, 1, 1, 64, [(1, 1, 64)] * w.heads, 1, 99))[0]
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    scores = torch.empty((w.B, w.heads, nt_cap, nt_cap), dtype=torch.float32, device=DEV)
    ws = torch.empty(V.veda_tile_scores_ws_bytes(L, 64) // 4, dtype=torch.float32, device=DEV)
    V.veda_tile_scores(L, T(dq), T(dk), T(w1), T(b1), T(w2), T(b2), T(w1k), T(b1), T(w2), T(b2), 128, 64,
                       synth.SCORE_SCALE, scores, ws)
    got = scores.cpu().numpy()
    for b in range(w.B):
        for h in range(w.heads):
            nt = lays[h]["nt"]
            ref = O.tile_scores(dq[b, h, :nt].astype(np.float64), dk[b, h, :nt].astype(np.float64), w1[h], b1[h],
                                w2[h], b2[h], w1k[h], b1[h], w2[h], b2[h], synth.SCORE_SCALE)
            _row_rel(got[b, h, :nt, :nt], ref)
            assert not got[b, h, nt:].any() and not got[b, h, :, nt:].any()


def _scores_topk_pair(w, zero_out=False, seed=5):
    """Unfused (scores, then top-k) and fused outputs on the same random
    descriptors and weights."""
    L = _layer(w)
    nt_cap = L.nt_cap
    rng = np.random.default_rng(seed)
    dq = rng.standard_normal((w.B, w.heads, nt_cap, 3 * w.d)).astype(np.float32)
    dk = rng.standard_normal((w.B, w.heads, nt_cap, 3 * w.d)).astype(np.float32)
    w1, b1, w2, b2 = synth.mlp_weights(w)
    b1 = rng.standard_normal(b1.shape).astype(np.float32) * 0.1
    b2 = rng.standard_normal(b2.shape).astype(np.float32) * 0.1
    if zero_out:                       # every score 0: the tie rule alone decides
        w2, b2 = np.zeros_like(w2), np.zeros_like(b2)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    args = [T(a) for a in (dq, dk, w1, b1, w2, b2, w1, b1, w2, b2)]
    ks = [max(1, (L.nt[h] * (h + 1)) // (3 * w.heads)) for h in range(w.heads)]
    k_cap = max(ks) + 2
    ws = torch.empty(V.veda_tile_scores_ws_bytes(L, 64) // 4, dtype=torch.float32, device=DEV)
    s1 = torch.empty((w.B, w.heads, nt_cap, nt_cap), dtype=torch.float32, device=DEV)
    i1 = torch.empty((w.B, w.heads, nt_cap, k_cap), dtype=torch.int32, device=DEV)
    m1 = torch.empty((w.B, w.heads, nt_cap, nt_cap), dtype=torch.uint8, device=DEV)
    V.veda_tile_scores(L, *args, 128, 64, synth.SCORE_SCALE, s1, ws)
    V.veda_topk_mask(L, s1, ks, k_cap, i1, m1)
    s2, i2, m2 = torch.full_like(s1, 7.0), torch.full_like(i1, 7), torch.full_like(m1, 7)
    V.veda_tile_scores_topk(L, *args, 128, 64, synth.SCORE_SCALE, ks, k_cap, i2, ws, mask=m2, scores=s2)
    i3 = torch.full_like(i1, 7)
    V.veda_tile_scores_topk(L, *args, 128, 64, synth.SCORE_SCALE, ks, k_cap, i3, ws)
    V.veda_check_status(L)
    return L, ks, k_cap, (s1, i1, m1), (s2, i2, m2), i3


@pytest.mark.parametrize("name", list(WL))
@pytest.mark.parametrize("zero_out", [False, True])
def test_tile_scores_topk_fused(name, zero_out):
    """The fused call gives bit-identical scores, index lists and mask to the
    two unfused calls (with and without the optional outputs), and its lists
    are the oracle's top-k of those scores."""
    w = WL[name]
    L, ks, k_cap, (s1, i1, m1), (s2, i2, m2), i3 = _scores_topk_pair(w, zero_out)
    assert torch.equal(s1, s2) and torch.equal(i1, i2) and torch.equal(m1, m2) and torch.equal(i1, i3)
    sc, gi = s1.cpu().numpy(), i2.cpu().numpy()
    for b in range(w.B):
        for h in range(w.heads):
            nt = L.nt[h]
            ri, _ = O.topk_rows(sc[b, h, :nt, :nt], ks[h], k_cap)
            assert np.array_equal(gi[b, h, :nt], ri)
            assert (gi[b, h, nt:] == -1).all()


def test_tile_scores_topk_fused_long_rows():
    """8,000 key tiles per row: fewer rows per CTA (6) fit shared memory."""
    w = synth.custom("long", 1, 2, 64, 8000, 8, 8, 64, [(1, 8, 8), (1, 8, 8)], 0.1, 31)
    L, ks, k_cap, (s1, i1, m1), (s2, i2, m2), i3 = _scores_topk_pair(w)
    assert torch.equal(s1, s2) and torch.equal(i1, i2) and torch.equal(m1, m2) and torch.equal(i1, i3)


# -------------------------------------------------------------------- top-k

def _topk_case(w, scores_np, k):
    L = _layer(w)
    nt_cap = L.nt_cap
    k_cap = max(k) + 3
    idx = torch.empty((w.B, w.heads, nt_cap, k_cap), dtype=torch.int32, device=DEV)
    mask = torch.empty((w.B, w.heads, nt_cap, nt_cap), dtype=torch.uint8, device=DEV)
    V.veda_topk_mask(L, torch.from_numpy(scores_np).to(DEV), k, k_cap, idx, mask)
    gi, gm = idx.cpu().numpy(), mask.cpu().numpy()
    for b in range(w.B):
        for h in range(w.heads):
            nt = L.nt[h]
            ri, rm = O.topk_rows(scores_np[b, h, :nt, :nt], k[h], k_cap)
            assert np.array_equal(gi[b, h, :nt], ri)
            assert np.array_equal(gm[b, h, :nt, :nt], rm)
            assert (gi[b, h, nt:] == -1).all() and not gm[b, h, nt:].any() and not gm[b, h, :, nt:].any()


@pytest.mark.parametrize("name", list(WL))
@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "signed-zero"])
def test_topk_bit_exact(name, kind):
    w = WL[name]
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    rng = np.random.default_rng(6)
    s = rng.standard_normal((w.B, w.heads, nt_cap, nt_cap)).astype(np.float32)
    if kind == "ties":
        s = np.round(s * 2) / 2
    elif kind == "zeros":
        s[:] = 0
    elif kind == "signed-zero":
        s = np.where(rng.random(s.shape) < 0.5, np.float32(-0.0), np.float32(0.0)).astype(np.float32)
        s[..., ::3] = 1.0
    ks = oracle_k(w, lays)
    _topk_case(w, s, ks)
    _topk_case(w, s, [1] * w.heads)
    _topk_case(w, s, [l["nt"] for l in lays])


def test_topk_large_rows():
    w = synth.sweep(261120, 0.03)      # 2040 tiles per row
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    rng = np.random.default_rng(7)
    s = (rng.standard_normal((1, w.heads, nt_cap, nt_cap)) * 3).astype(np.float32)
    s = np.round(s * 64) / 64                              # frequent ties
    _topk_case(w, s, oracle_k(w, lays))


def test_topk_rows_past_register_path():
    """Rows longer than 2048 tiles take the shared-memory radix selection."""
    w = synth.custom("rows2112-d64-t64", 1, 2, 64, 33, 64, 64, 64, [(1, 8, 8), (1, 8, 8)], 0.1, 9)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    assert nt_cap == 2112
    rng = np.random.default_rng(8)
    s = (rng.standard_normal((1, w.heads, nt_cap, nt_cap)) * 3).astype(np.float32)
    s = np.round(s * 64) / 64                              # frequent ties
    _topk_case(w, s, oracle_k(w, lays))
    _topk_case(w, s, [1, nt_cap])


# --------------------------------------------------------- sparse attention

def _attention_case(w, k_override=None, dense=False, random_lists=True, key_tile_gain=None, shuffle=False):
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, k, v = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    vp, _ = _permuted(L, w, v)
    if key_tile_gain is not None:       # per key tile factor on K (and so on its logits)
        for h in range(w.heads):
            g = key_tile_gain(lays[h]["nt"])
            for t, f in enumerate(g):
                kp[:, h, t * w.tile:(t + 1) * w.tile] = (kp[:, h, t * w.tile:(t + 1) * w.tile].float() * f).bfloat16()
    ks = k_override or oracle_k(w, lays)
    k_cap = max(ks)
    idx = np.full((w.B, w.heads, nt_cap, k_cap), -1, np.int32)
    for b in range(w.B):
        for h in range(w.heads):
            nt = lays[h]["nt"]
            idx[b, h, :nt] = synth.random_index_lists(nt, nt, ks[h], k_cap, seed=100 * b + h + w.seed)
            if shuffle:     # kept tiles in any order: the same attention
                rng = np.random.default_rng(500 + 100 * b + h)
                for a in range(nt):
                    idx[b, h, a, :ks[h]] = rng.permutation(idx[b, h, a, :ks[h]])
    op = torch.empty_like(qp)
    lse = torch.empty((w.B, w.heads, n_cap), dtype=torch.float32, device=DEV)
    scale = 1 / math.sqrt(w.d)
    if dense:
        V.veda_sparse_attn(L, qp, kp, vp, None, None, 0, scale, op, lse)
    else:
        V.veda_sparse_attn(L, qp, kp, vp, torch.from_numpy(idx).to(DEV), ks, k_cap, scale, op, lse)
    V.veda_check_status(L)
    go, gl = f64(op), lse.cpu().double().numpy()
    xq, xk, xv = f64(qp), f64(kp), f64(vp)
    for b in range(w.B):
        for h in range(w.heads):
            nt, lens = lays[h]["nt"], lays[h]["lens"]
            ih = np.tile(np.arange(nt), (nt, 1)) if dense else idx[b, h, :nt]
            kk = nt if dense else ks[h]
            ref = O.sparse_attention(xq[b, h], xk[b, h], xv[b, h], ih, kk, lens, w.tile, scale)
            _check_attention(go[b, h], gl[b, h], ref, lens, w.tile)
            # padding rows and tiles beyond nt are zero
            for a in range(nt):
                assert not go[b, h, a * w.tile + lens[a]:(a + 1) * w.tile].any()
            assert not go[b, h, nt * w.tile:].any()


@pytest.mark.parametrize("name", list(WL))
def test_sparse_attention_random_lists(name):
    _attention_case(WL[name])


@pytest.mark.parametrize("name", ["ragged-d128-t128", "batch2-d64-t128", "odd-d128-t64"])
def test_sparse_attention_unsorted_lists(name):
    """Kept-tile lists in arbitrary order (the call does not require them
    ascending): the kernel then merges the lists instead of walking its
    kept-tile bitmaps, with the same result."""
    _attention_case(WL[name], shuffle=True)


@pytest.mark.parametrize("name", list(WL))
@pytest.mark.parametrize("dense", [False, True])
def test_sparse_attention_unpermute_fused(name, dense):
    """veda_sparse_attn_unpermute writes each output row straight to its
    token: bit-identical to veda_sparse_attn followed by the inverse
    permutation (every token written), the same lse. veda_sparse_attn_tokens
    (Q, K, V gathered from token order by TMA) gives the same output and lse."""
    w = WL[name]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, k, v = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    vp, _ = _permuted(L, w, v)
    ks = oracle_k(w, lays)
    k_cap = max(ks)
    idx = np.full((w.B, w.heads, nt_cap, k_cap), -1, np.int32)
    for b in range(w.B):
        for h in range(w.heads):
            nt = lays[h]["nt"]
            idx[b, h, :nt] = synth.random_index_lists(nt, nt, ks[h], k_cap, seed=300 + 100 * b + h + w.seed)
    idx_d = None if dense else torch.from_numpy(idx).to(DEV)
    args = (None, None, 0) if dense else (idx_d, ks, k_cap)
    scale = 1 / math.sqrt(w.d)
    op = torch.empty_like(qp)
    lse1 = torch.empty((w.B, w.heads, n_cap), dtype=torch.float32, device=DEV)
    V.veda_sparse_attn(L, qp, kp, vp, *args, scale, op, lse1)
    o_sep = torch.full_like(q, 3.0)
    V.veda_permute(L, o_sep, op, inverse=True)
    o = torch.full_like(q, 7.0)                       # every token must be overwritten
    lse2 = torch.empty_like(lse1)
    V.veda_sparse_attn_unpermute(L, qp, kp, vp, *args, scale, o, lse2)
    # and with no permuted copies at all: tiles gathered by TMA from token order
    o3 = torch.full_like(q, 5.0)
    lse3 = torch.empty_like(lse1)
    V.veda_sparse_attn_tokens(L, q, k, v, *args, scale, o3, lse3)
    V.veda_check_status(L)
    torch.cuda.synchronize()
    assert torch.equal(o, o_sep)
    assert torch.equal(lse1, lse2)
    assert torch.equal(o3, o_sep)
    assert torch.equal(lse3, lse1)          # padding rows are 0 on both paths


@pytest.mark.parametrize("name", list(WL))
def test_sparse_attention_dense_path(name):
    _attention_case(WL[name], dense=True)


@pytest.mark.parametrize("name", ["ragged-d128-t128", "odd-d128-t64"])
def test_sparse_attention_k1_and_keep_all(name):
    w = WL[name]
    lays, _, _, _ = oracle_geometry(w)
    _attention_case(w, k_override=[1] * w.heads)
    _attention_case(w, k_override=[l["nt"] for l in lays])


@pytest.mark.parametrize("name", ["ragged-d128-t128", "batch2-d64-t128", "odd-d128-t64"])
@pytest.mark.parametrize("order", ["growing", "shrinking"])
def test_sparse_attention_wide_logit_range(name, order):
    """Key tiles whose logits differ by hundreds of units: with `growing`, every
    later kept tile out-scores the first one far beyond the fp32 exponent range
    unless the running reference moves; with `shrinking`, later tiles
    underflow against the first. Both must match the oracle's exact softmax."""
    def gain(nt):
        f = 1.0 + 6.0 * np.arange(nt)
        return f if order == "growing" else f[::-1]
    _attention_case(WL[name], key_tile_gain=gain)
    _attention_case(WL[name], dense=True, key_tile_gain=gain)


@pytest.mark.parametrize("name", list(WL))
@pytest.mark.parametrize("dense", [False, True])
def test_sparse_attention_deterministic(name, dense):
    """Repeated calls give the same bits: the kernels sum in a fixed order, so
    any difference is a race (a buffer read before the MMA or softmax that
    writes it has finished)."""
    w = WL[name]
    L = _layer(w)
    lays, _, _, nt_cap = oracle_geometry(w)
    q, k, v = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    vp, _ = _permuted(L, w, v)
    ks = oracle_k(w, lays)
    k_cap = max(ks)
    idx = np.full((w.B, w.heads, nt_cap, k_cap), -1, np.int32)
    for b in range(w.B):
        for h in range(w.heads):
            nt = lays[h]["nt"]
            idx[b, h, :nt] = synth.random_index_lists(nt, nt, ks[h], k_cap, seed=7 + 100 * b + h)
    idx_d = torch.from_numpy(idx).to(DEV)
    outs = []
    for _ in range(4):
        op = torch.zeros_like(qp)
        if dense:
            V.veda_sparse_attn(L, qp, kp, vp, None, None, 0, 0.1, op)
        else:
            V.veda_sparse_attn(L, qp, kp, vp, idx_d, ks, k_cap, 0.1, op)
        outs.append(op)
    torch.cuda.synchronize()
    V.veda_check_status(L)
    for o in outs[1:]:
        assert torch.equal(outs[0], o)


def test_sparse_attention_bad_index_reported():
    w = WL["ragged-d128-t128"]
    L = _layer(w)
    q, k, v = _inputs(w)
    qp, _ = _permuted(L, w, q)
    idx = torch.zeros((1, w.heads, L.nt_cap, 2), dtype=torch.int32, device=DEV)
    idx[0, 1, 0, 1] = 10_000
    op = torch.empty_like(qp)
    V.veda_sparse_attn(L, qp, qp, qp, idx, [2] * w.heads, 2, 0.1, op)
    with pytest.raises(V.VedaError) as e:
        V.veda_check_status(L)
    assert e.value.code == V.VEDA_ERR_BAD_INDEX
    V.veda_check_status(L)      # cleared


# ----------------------------------------------------- tile map, lse and KL

@pytest.mark.parametrize("name", list(WL))
def test_tilemap_lse_kl(name):
    w = WL[name]
    if w.B != 1:
        pytest.skip("tile map is defined for B == 1 layers")
    _tilemap_case(w)


@pytest.mark.parametrize("name", ["ragged-d128-t128", "odd-d128-t64", "d64-t64-padded"])
@pytest.mark.parametrize("order", ["growing", "shrinking"])
def test_tilemap_wide_logit_range(name, order):
    """Key tiles whose logits differ by hundreds of units (as in the attention
    case): the row log-sum-exp must move its reference when a later key tile
    out-scores the first one beyond the fp32 exponent range."""
    def gain(nt):
        f = 1.0 + 6.0 * np.arange(nt)
        return f if order == "growing" else f[::-1]
    _tilemap_case(WL[name], key_tile_gain=gain)


def _tilemap_case(w, key_tile_gain=None):
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, k, _ = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    if key_tile_gain is not None:
        for h in range(w.heads):
            for t, f in enumerate(key_tile_gain(lays[h]["nt"])):
                kp[:, h, t * w.tile:(t + 1) * w.tile] = (kp[:, h, t * w.tile:(t + 1) * w.tile].float() * f).bfloat16()
    heads = list(range(w.heads))
    n_rows = min(l["nt"] for l in lays)
    rows = np.stack([np.sort(np.random.default_rng(h).choice(lays[h]["nt"], n_rows, replace=False))
                     for h in heads]).astype(np.int32)
    rng = np.random.default_rng(8)
    scores = rng.standard_normal((1, w.heads, nt_cap, nt_cap)).astype(np.float32)
    tm = torch.empty((len(heads), n_rows, nt_cap), dtype=torch.float32, device=DEV)
    lse = torch.empty((len(heads), n_rows, w.tile), dtype=torch.float32, device=DEV)
    klr = torch.empty((len(heads), n_rows), dtype=torch.float32, device=DEV)
    klo = torch.empty(4, dtype=torch.float32, device=DEV)
    scale = 1 / math.sqrt(w.d)
    V.veda_full_attn_tilemax(L, qp, kp, heads, torch.from_numpy(rows).to(DEV), n_rows, scale, tm, lse,
                             torch.from_numpy(scores).to(DEV), klr, klo)
    V.veda_check_status(L)
    gm, gl, gk = tm.cpu().double().numpy(), lse.cpu().double().numpy(), klr.cpu().double().numpy()
    xq, xk = f64(qp), f64(kp)
    kl_heads = []
    for s, h in enumerate(heads):
        nt, lens = lays[h]["nt"], lays[h]["lens"]
        M, lse_ref = O.full_tilemap(xq[0, h], xk[0, h], lens, w.tile, scale, rows[s])
        _row_rel(gm[s, :, :nt], M)
        assert not gm[s, :, nt:].any()
        for r, a in enumerate(rows[s]):
            np.testing.assert_allclose(gl[s, r, :lens[a]], lse_ref[a], rtol=1e-4, atol=1e-4)
        kl = O.kl_rows(M, scores[0, h, rows[s]][:, :nt])
        np.testing.assert_allclose(gk[s], kl, rtol=1e-3, atol=1e-5)
        kl_heads.append(kl.mean())
    assert float(klo[0]) == pytest.approx(float(np.mean(kl_heads)), rel=1e-3)


def test_tilemap_all_rows_default_list():
    w = WL["cfg0"]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, k, _ = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    tm = torch.empty((2, 4, nt_cap), dtype=torch.float32, device=DEV)
    V.veda_full_attn_tilemax(L, qp, kp, [1, 0], None, 4, 0.125, tm)
    gm = tm.cpu().double().numpy()
    for s, h in enumerate([1, 0]):
        M, _ = O.full_tilemap(f64(qp)[0, h], f64(kp)[0, h], lays[h]["lens"], w.tile, 0.125)
        _row_rel(gm[s], M)


@pytest.mark.parametrize("idx,heads,n_rows", [(1, [3, 7], 6), (2, [0], 5), (4, [1, 5], 9)])
def test_tilemap_split_key_range(idx, heads, n_rows):
    """With a workspace the map may split each row pair's key range over
    several CTAs (partial sums, then a fixed-order combination): same map,
    log-sum-exp and KL as the single-CTA path, and the oracle's values on the
    rows checked. Layers: 24,576 tokens with 64-token tiles, 80,640 tokens
    with padded T, 65,280 tokens."""
    w = synth.config(idx)
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, k, _ = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    rng = np.random.default_rng(11)
    rows = np.stack([np.sort(rng.choice(lays[h]["nt"], n_rows, replace=False)) for h in heads]).astype(np.int32)
    rows_d = torch.from_numpy(rows).to(DEV)
    scores = torch.from_numpy(rng.standard_normal((1, w.heads, nt_cap, nt_cap)).astype(np.float32)).to(DEV)
    scale = 1 / math.sqrt(w.d)
    out = {}
    for use_ws in (False, True):
        tm = torch.full((len(heads), n_rows, nt_cap), 7.0, dtype=torch.float32, device=DEV)
        lse = torch.full((len(heads), n_rows, w.tile), 7.0, dtype=torch.float32, device=DEV)
        klr = torch.empty((len(heads), n_rows), dtype=torch.float32, device=DEV)
        klo = torch.empty(4, dtype=torch.float32, device=DEV)
        ws = None
        if use_ws:
            ws = torch.empty(V.veda_full_attn_tilemax_ws_bytes(L, len(heads), n_rows) // 4, dtype=torch.float32,
                             device=DEV)
        V.veda_full_attn_tilemax(L, qp, kp, heads, rows_d, n_rows, scale, tm, lse, scores, klr, klo, ws=ws)
        V.veda_check_status(L)
        out[use_ws] = [t.cpu().double().numpy() for t in (tm, lse, klr, klo[:1])]
        # the KL of the finished map, taken separately, is the same
        klr2, klo2 = torch.empty_like(klr), torch.empty_like(klo)
        V.veda_tilemap_kl(L, heads, rows_d, n_rows, tm, scores, klr2, klo2)
        torch.cuda.synchronize()
        assert torch.equal(klr2, klr) and torch.equal(klo2[:1], klo[:1])
    for a, b in zip(out[False], out[True]):
        np.testing.assert_allclose(b, a, rtol=1e-5, atol=1e-30)
    gm = out[True][0]
    for s, h in enumerate(heads):
        nt = lays[h]["nt"]
        pick = [0, n_rows - 1]
        M, _ = O.full_tilemap(f64(qp)[0, h], f64(kp)[0, h], lays[h]["lens"], w.tile, scale, rows[s, pick])
        _row_rel(gm[s, pick, :nt], M)
        assert not gm[s, :, nt:].any()


# ------------------------------------------------ recall of the mask (a9)

def _recall_rows_oracle(pred_idx, M_rows, k):
    """Hits per row through the oracle's recall on single rows."""
    nt = M_rows.shape[1]
    out = []
    for p, m in zip(pred_idx, M_rows):
        mask = np.zeros((1, nt), bool)
        mask[0, p[:k]] = True
        out.append(round(O.recall(mask, m[None], k) * k))
    return np.array(out)


@pytest.mark.parametrize("name", ["cfg0", "ragged-d128-t128", "odd-d128-t64", "d64-t64-padded", "single-tile"])
@pytest.mark.parametrize("kmode", ["keep", "one", "all"])
def test_tilemap_recall(name, kmode):
    """Recall of a predicted top-k mask against the tile map's own top-k
    (Veda summary 2.1, Target Construction). Exact against the oracle's
    recall applied to the GPU's map rows and mask (hits are integers; the map
    is ranked with the same fp32 order and tie rule), and equal to the
    oracle's recall on the fp64 oracle map wherever that row's top-k is not
    decided by values closer than the map tolerance (1e-3 relative)."""
    w = WL[name]
    L = _layer(w)
    lays, perms, n_cap, nt_cap = oracle_geometry(w)
    q, k, _ = _inputs(w)
    qp, _ = _permuted(L, w, q)
    kp, _ = _permuted(L, w, k)
    heads = list(range(w.heads))[::-1]
    n_rows = min(l["nt"] for l in lays)
    rows = np.stack([np.random.default_rng(30 + h).permutation(lays[h]["nt"])[:n_rows] for h in heads]).astype(np.int32)
    kk = {"keep": oracle_k(w, lays), "one": [1] * w.heads, "all": [l["nt"] for l in lays]}[kmode]
    k_cap = max(kk)
    scale = 1 / math.sqrt(w.d)
    tm = torch.empty((len(heads), n_rows, nt_cap), dtype=torch.float32, device=DEV)
    rows_d = torch.from_numpy(rows).to(DEV)
    V.veda_full_attn_tilemax(L, qp, kp, heads, rows_d, n_rows, scale, tm)
    # the predicted lists: top-k of random scores with planted ties
    rng = np.random.default_rng(9)
    sc = rng.integers(0, 4, size=(1, w.heads, nt_cap, nt_cap)).astype(np.float32)
    idx = torch.empty((1, w.heads, nt_cap, k_cap), dtype=torch.int32, device=DEV)
    V.veda_topk_mask(L, torch.from_numpy(sc).to(DEV), kk, k_cap, idx)
    hits = torch.full((len(heads), n_rows), -7, dtype=torch.int32, device=DEV)
    rec = torch.empty(len(heads) + 1, dtype=torch.float32, device=DEV)
    map_idx = torch.empty((len(heads), n_rows, k_cap), dtype=torch.int32, device=DEV)
    V.veda_tilemap_recall(L, heads, rows_d, n_rows, tm, idx, kk, k_cap, hits, rec, map_idx=map_idx)
    V.veda_check_status(L)
    gm = tm.cpu().numpy()
    gh, gr, gi = hits.cpu().numpy(), rec.cpu().numpy().astype(np.float64), map_idx.cpu().numpy()
    pred_all = idx.cpu().numpy()
    xq, xk = f64(qp), f64(kp)
    per_head = []
    for s, h in enumerate(heads):
        nt, kh = lays[h]["nt"], kk[h]
        pred = pred_all[0, h, rows[s]]
        # exact: the oracle's ranking of the GPU's fp32 map rows
        ref_idx, _ = O.topk_rows(gm[s, :, :nt], kh, k_cap)
        assert np.array_equal(gi[s], ref_idx)
        want = _recall_rows_oracle(pred, gm[s, :, :nt], kh)
        assert np.array_equal(gh[s], want)
        mask = np.zeros((n_rows, nt), bool)
        for r in range(n_rows):
            mask[r, pred[r, :kh]] = True
        r_or = O.recall(mask, gm[s, :, :nt], kh)
        assert gr[s] == pytest.approx(r_or, abs=1e-6)
        per_head.append(r_or)
        # against the fp64 oracle map, on rows whose top-k is not a near tie
        M, _ = O.full_tilemap(xq[0, h], xk[0, h], lays[h]["lens"], w.tile, scale, rows[s])
        want64 = _recall_rows_oracle(pred, M, kh)
        srt = -np.sort(-M, axis=1)
        clear = np.ones(n_rows, bool) if kh >= nt else (srt[:, kh - 1] - srt[:, kh]) > 1e-3 * srt[:, 0]
        assert clear.any()
        assert np.array_equal(gh[s][clear], want64[clear])
    assert gr[-1] == pytest.approx(np.mean(per_head), abs=1e-6)
    if kmode == "all":
        assert (gh == np.array([[kk[h]] for h in heads])).all() and np.allclose(gr, 1.0)
