"""Estimator training on the GPU: the weight gradient of the distillation
loss (veda_estimator_grad) against the fp64 oracle (estimator_grad, pinned by
finite differences in test_oracle.py), on small layers, on sampled query
tiles, with the tile map from the library's own kernel and with random maps.

Tolerance: each gradient array within 1e-4 of the largest oracle gradient
of its side. The GPU sums up to nt * rows fp32 terms per weight in a fixed
order (unit roundoff u = 6e-8); for terms of mixed sign the error grows like
sqrt(n) * u, about 2e-5 of the largest term at n = 1.4e5 (the 153,600-token
layer's 120 rows x 1,200 tiles), and the largest observed on these layers
was 1e-5. The loss within 1e-4 relative."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_24_b200 as V
import synth
from oracle import veda_oracle as O
from tests.helpers import f64, oracle_geometry, small_workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
WL = {n: w for n, w in small_workloads().items() if w.B == 1}
NAMES = ["w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k"]


def _weights(w, seed, tied):
    rng = np.random.default_rng(seed)
    w1, b1, w2, b2 = synth.mlp_weights(w)
    b1 = rng.standard_normal(b1.shape).astype(np.float32) * 0.1
    b2 = rng.standard_normal(b2.shape).astype(np.float32) * 0.1
    if tied:
        return [w1, b1, w2, b2, w1, b1, w2, b2]
    w1k = (w1 * rng.uniform(0.5, 1.5, w1.shape)).astype(np.float32)
    w2k = (w2 * rng.uniform(0.5, 1.5, w2.shape)).astype(np.float32)
    return [w1, b1, w2, b2, w1k, b1 * 0.5, w2k, b2 * 2.0]


def _case(w, heads, n_rows, map_kind, tied=False, seed=0):
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device=DEV)
    lays, _, n_cap, nt_cap = oracle_geometry(w)
    rng = np.random.default_rng(seed)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    q, k, _ = (t.to(DEV) for t in synth.qkv(w, "cpu"))
    qp = torch.empty((1, w.heads, n_cap, w.d), dtype=torch.bfloat16, device=DEV)
    kp = torch.empty_like(qp)
    dq = torch.empty((1, w.heads, nt_cap, 3 * w.d), dtype=torch.float32, device=DEV)
    dk = torch.empty_like(dq)
    V.veda_permute_trippool(L, q, qp, dq)
    V.veda_permute_trippool(L, k, kp, dk)
    rows = np.stack([np.sort(rng.choice(lays[h]["nt"], n_rows, replace=False)) for h in heads]).astype(np.int32)
    tm = torch.empty((len(heads), n_rows, nt_cap), dtype=torch.float32, device=DEV)
    if map_kind == "tilemap":
        V.veda_full_attn_tilemax(L, qp, kp, heads, T(rows), n_rows, 1 / math.sqrt(w.d), tm)
    else:
        m = rng.uniform(0.0, 1.0, (len(heads), n_rows, nt_cap)).astype(np.float32)
        m[m < 0.2] = 0.0
        for s, h in enumerate(heads):
            m[s, :, lays[h]["nt"]:] = 0.0
            m[s, :, 0] = 0.5                      # every row has mass
        tm.copy_(T(m))
    Wn = _weights(w, seed + 1, tied)
    Wt = [T(a) for a in Wn]
    grads = [torch.full_like(t, 7.0) for t in Wt]  # poisoned: every entry must be written
    loss = torch.full((1,), 7.0, dtype=torch.float32, device=DEV)
    ws = torch.empty(V.veda_estimator_grad_ws_bytes(L, len(heads), n_rows, 128, 64) // 4, dtype=torch.float32,
                     device=DEV)
    scale = synth.SCORE_SCALE
    V.veda_estimator_grad(L, dq, dk, Wt, 128, 64, scale, heads, T(rows), n_rows, tm, grads, ws, loss)
    V.veda_check_status(L)
    got = [g.cpu().double().numpy() for g in grads]
    # oracle: per selected head, gradient of that head's mean-over-rows loss,
    # scaled by 1/heads (mean over heads); zero for the other heads
    ref = [np.zeros_like(a, dtype=np.float64) for a in Wn]
    xq, xk, M = f64(dq)[0], f64(dk)[0], tm.cpu().double().numpy()
    losses = []
    for s, h in enumerate(heads):
        nt = lays[h]["nt"]
        args = [a[h].astype(np.float64) for a in Wn]
        g = O.estimator_grad(xq[h, rows[s]], xk[h, :nt], *args, scale, M[s, :, :nt])
        for i, n in enumerate(NAMES):
            ref[i][h] = g[n] / len(heads)
        losses.append(O.estimator_loss(xq[h, rows[s]], xk[h, :nt], *args, scale, M[s, :, :nt]))
    for side in (0, 1):
        scale_side = max(np.abs(ref[4 * side + i]).max() for i in range(4))
        for i in range(4 * side, 4 * side + 4):
            err = np.abs(got[i] - ref[i]).max()
            assert err <= 1e-4 * scale_side, (NAMES[i], err, scale_side)
    assert float(loss.item()) == pytest.approx(float(np.mean(losses)), rel=1e-4)
    return L, (dq, dk, Wt, heads, T(rows), n_rows, tm, ws), grads


@pytest.mark.parametrize("name", list(WL))
@pytest.mark.parametrize("map_kind", ["tilemap", "random"])
def test_estimator_grad_matches_oracle(name, map_kind):
    w = WL[name]
    lays, _, _, _ = oracle_geometry(w)
    n_rows = min(3, min(l["nt"] for l in lays))
    heads = list(range(w.heads))[::-1][: max(1, w.heads - 1)]   # a subset, in a non-sorted order
    _case(w, heads, n_rows, map_kind)


def test_estimator_grad_tied_weights_and_determinism():
    """One MLP for both sides (the layer's use): the two gradients are each
    the oracle's; two calls are bit-identical."""
    w = WL["ragged-d128-t128"]
    L, args, grads = _case(w, [1, 3], 2, "tilemap", tied=True)
    dq, dk, Wt, heads, rows, n_rows, tm, ws = args
    again = [torch.empty_like(g) for g in grads]
    V.veda_estimator_grad(L, dq, dk, Wt, 128, 64, synth.SCORE_SCALE, heads, rows, n_rows, tm, again, ws)
    torch.cuda.synchronize()
    for a, b in zip(grads, again):
        assert torch.equal(a, b)


def test_estimator_grad_argument_checks():
    w = WL["cfg0"]
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device=DEV)
    z = torch.zeros(1024, dtype=torch.float32, device=DEV)
    with pytest.raises(V.VedaError) as e:
        V.veda_estimator_grad(L, z, z, [z] * 8, 128, 64, 0.125, [0, 0], None, 1, z, [z] * 8, z)
    assert e.value.code == V.VEDA_ERR_INVALID_ARG and "twice" in str(e.value)
    with pytest.raises(V.VedaError) as e:
        V.veda_estimator_grad(L, z, z, [z] * 8, 130, 64, 0.125, [0], None, 1, z, [z] * 8, z)
    assert e.value.code == V.VEDA_ERR_UNSUPPORTED
