"""Full-size parity: the benchmark's layers, built and launched exactly as
bench.py does, checked against the fp64 oracle on sampled outputs.

Per layer: the permutation map of every head is compared whole; permuted and
un-permuted rows, TripPool tiles, score rows, top-k rows (all of them),
attention query tiles, tile-map rows and KL rows are compared on seeded
samples, each stage on the GPU's own upstream values (the oracle ranks the
GPU's fp32 scores and attends over the GPU's index lists). Tolerances as in
test_gpu_parity.py."""
import math

import numpy as np
import pytest
import torch

import bench
import synth
from oracle import veda_oracle as O

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _row_rel(got, want, tol=1e-3):
    for g, w_ in zip(np.atleast_2d(got), np.atleast_2d(want)):
        scale = max(np.abs(w_).max(), 1e-30)
        assert np.abs(g - w_).max() <= tol * scale, (np.abs(g - w_).max(), scale)


WORKLOADS = {
    "24576tok-tile64": lambda: synth.config(1),
    "80640tok-padded-T": lambda: synth.config(2),
    "153600tok-90pct": lambda: synth.config(3),
    "153600tok-95pct": lambda: synth.config(3, keep=0.05),
    "261120tok-97pct": lambda: synth.sweep(261120, 0.03),
}


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_layer_sampled(name):
    w = WORKLOADS[name]()
    V, L, layer, (q, k, v) = bench.build_layer(w, DEV)
    layer.forward(q, k, v)
    V.veda_check_status(L)
    torch.cuda.synchronize()
    rng = np.random.default_rng(123)
    heads = sorted(set([0, w.heads - 1] + list(rng.choice(w.heads, size=min(3, w.heads), replace=False))))
    np_w = synth.mlp_weights(w)
    perm_gpu = layer.perm.cpu().numpy()
    scale = 1 / math.sqrt(w.d)

    for h in range(w.heads):                               # permutation maps: every head, whole
        p = O.perm_indices(w.T, w.H, w.W, w.tilings[h])
        assert np.array_equal(perm_gpu[h, :len(p)], p)
        assert (perm_gpu[h, len(p):] == -1).all()

    for h in heads:
        lay = O.head_layout(w.T, w.H, w.W, w.tilings[h])
        nt, lens = lay["nt"], lay["lens"]
        perm = O.perm_indices(w.T, w.H, w.W, w.tilings[h])
        # permuted rows: bit-exact on sampled slots of Q, K and V
        slots = rng.choice(np.nonzero(perm >= 0)[0], size=min(4096, int((perm >= 0).sum())), replace=False)
        for src, dst in ((q, layer.qp), (k, layer.kp), (v, layer.vp)):
            got = dst[0, h, torch.from_numpy(slots).to(DEV)]
            want = src[0, torch.from_numpy(perm[slots]).to(DEV), h]
            assert torch.equal(got, want)
        qp, kp, vp = (_f64(t[0, h]) for t in (layer.qp, layer.kp, layer.vp))

        # TripPool on sampled tiles
        tiles = np.unique(np.concatenate([[0, nt - 1], rng.choice(nt, size=min(32, nt), replace=False)]))
        dq_all, dk_all = _f64(layer.dq[0, h]), _f64(layer.dk[0, h])
        for src, got in ((qp, dq_all), (kp, dk_all)):
            ref = O.trippool(src, lens, w.tile)
            np.testing.assert_allclose(got[tiles, :w.d], ref[tiles, :w.d], rtol=1e-6, atol=1e-6)
            assert np.array_equal(got[tiles, w.d:], ref[tiles, w.d:])

        # tile scores from the GPU's descriptors, all rows of the head
        w1, b1, w2, b2 = (a[h] for a in np_w)
        s_ref = O.tile_scores(dq_all[:nt], dk_all[:nt], w1, b1, w2, b2, w1, b1, w2, b2, synth.SCORE_SCALE)
        s_gpu = layer.scores[0, h, :nt, :nt].cpu().numpy()
        _row_rel(s_gpu, s_ref)

        # top-k of the GPU's fp32 scores: every row bit-exact
        kk = layer.k[h]
        idx_ref, mask_ref = O.topk_rows(s_gpu, kk, layer.k_cap)
        assert np.array_equal(layer.idx[0, h, :nt].cpu().numpy(), idx_ref)
        assert np.array_equal(layer.mask[0, h, :nt, :nt].cpu().numpy(), mask_ref)

        # sparse attention on sampled query tiles (first, last and random):
        # the layer's output is in token order, row i of tile a at token perm[a*tile + i]
        rows = np.unique(np.concatenate([[0, nt - 1], rng.choice(nt, size=min(6, nt), replace=False)]))
        ref = O.sparse_attention(qp, kp, vp, idx_ref, kk, lens, w.tile, scale, rows=rows)
        errs = []
        for a, (oa, _) in ref.items():
            toks_a = torch.from_numpy(perm[a * w.tile: a * w.tile + lens[a]]).to(DEV)
            errs.append(np.abs(_f64(layer.o[0, toks_a, h]) - oa).ravel())
        e = np.concatenate(errs)
        assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())

    # the fused token-order output equals the permuted output of the separate
    # call followed by the inverse permutation, bit for bit, on every token
    layer.attend_permuted()
    o_sep = torch.empty_like(layer.o)
    V.veda_permute(L, o_sep, layer.op, inverse=True)
    torch.cuda.synchronize()
    assert torch.equal(layer.o, o_sep)
    # and a second launch repeats the first bit for bit (a race between the
    # kernel's roles would show here first: thousands of CTAs)
    op_first = layer.op.clone()
    layer.attend_permuted()
    torch.cuda.synchronize()
    assert torch.equal(layer.op, op_first)

    # tile map and KL on the benchmark's sampled heads and query tiles
    m = layer.maps
    rows_all = m.rows.cpu().numpy()
    tm, klr = layer.tilemap.cpu().double().numpy(), layer.kl_rows.cpu().double().numpy()
    for s, h in enumerate(m.heads):
        lay = O.head_layout(w.T, w.H, w.W, w.tilings[h])
        nt, lens = lay["nt"], lay["lens"]
        qp, kp = _f64(layer.qp[0, h]), _f64(layer.kp[0, h])
        pick = np.unique(np.concatenate([[0, m.n_rows - 1], rng.choice(m.n_rows, size=4, replace=False)]))
        M, _ = O.full_tilemap(qp, kp, lens, w.tile, scale, rows_all[s, pick])
        _row_rel(tm[s, pick, :nt], M)
        s_gpu = layer.scores[0, h, :nt, :nt].cpu().numpy()
        kl = O.kl_rows(M, s_gpu[rows_all[s, pick]])
        np.testing.assert_allclose(klr[s, pick], kl, rtol=1e-3, atol=1e-5)
        # recall of the predicted mask against the map's top-k, every sampled
        # row: exact against the oracle's recall on the GPU's map rows
        kk = layer.k[h]
        mask = layer.mask[0, h, rows_all[s], :nt].cpu().numpy().astype(bool)
        hits = layer.recall_hits[s].cpu().numpy()
        for r in range(m.n_rows):
            assert hits[r] == round(O.recall(mask[r:r + 1], tm[s, r:r + 1, :nt].astype(np.float32), kk) * kk)
        assert float(layer.recall[s]) == pytest.approx(O.recall(mask, tm[s, :, :nt].astype(np.float32), kk),
                                                       abs=1e-6)


def test_dense_path_full_size_sampled():
    """The library's own dense path (every tile kept) at the 153,600-token
    layer, against textbook full attention on sampled query tiles."""
    w = synth.config(3)
    V, L, layer, (q, k, v) = bench.build_layer(w, DEV)
    layer.front(q, k, v)
    out = torch.empty_like(layer.op)
    layer.dense(out)
    V.veda_check_status(L)
    rng = np.random.default_rng(7)
    for h in (0, w.heads - 1):
        lay = O.head_layout(w.T, w.H, w.W, w.tilings[h])
        nt, lens = lay["nt"], lay["lens"]
        qp, kp, vp = (_f64(t[0, h]) for t in (layer.qp, layer.kp, layer.vp))
        rows = np.unique(np.concatenate([[0, nt - 1], rng.choice(nt, size=2, replace=False)]))
        ref = O.sparse_attention(qp, kp, vp, np.tile(np.arange(nt), (nt, 1)), nt, lens, w.tile,
                                 1 / math.sqrt(w.d), rows=rows)
        op = _f64(out[0, h])
        e = np.concatenate([np.abs(op[a * w.tile: a * w.tile + lens[a]] - oa).ravel() for a, (oa, _) in ref.items()])
        assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())


def test_estimator_grad_full_size():
    """The weight gradient of the distillation loss at the 153,600-token
    layer (2 heads x 120 sampled query tiles over 1,200 key tiles) against the
    fp64 oracle, from the layer's own descriptors and tile map."""
    w = synth.config(3)
    V, L, layer, (q, k, v) = bench.build_layer(w, DEV)
    layer.forward(q, k, v)
    grads, loss = layer.estimator_grad()
    V.veda_check_status(L)
    m = layer.maps
    rows = m.rows.cpu().numpy()
    xq, xk = _f64(layer.dq[0]), _f64(layer.dk[0])
    M = layer.tilemap.cpu().double().numpy()
    np_w = synth.mlp_weights(w)
    names = ["w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k"]
    got = [g.cpu().double().numpy() for g in grads]
    losses = []
    for s, h in enumerate(m.heads):
        nt = L.nt[h]
        args = [a[h].astype(np.float64) for a in np_w] * 2
        g = O.estimator_grad(xq[h, rows[s]], xk[h, :nt], *args, synth.SCORE_SCALE, M[s, :, :nt])
        losses.append(O.estimator_loss(xq[h, rows[s]], xk[h, :nt], *args, synth.SCORE_SCALE, M[s, :, :nt]))
        for side in (0, 1):
            scale = max(np.abs(g[n]).max() for n in names[4 * side: 4 * side + 4]) / len(m.heads)
            for i in range(4 * side, 4 * side + 4):
                err = np.abs(got[i][h] - g[names[i]] / len(m.heads)).max()
                assert err <= 1e-4 * scale, (names[i], h, err, scale)   # as in test_gpu_estimator.py
    for h in set(range(w.heads)) - set(m.heads):
        assert not any(got[i][h].any() for i in range(8))
    assert float(loss.item()) == pytest.approx(float(np.mean(losses)), rel=1e-4)
