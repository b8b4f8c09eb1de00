"""Temporal caching of tile scores (the library's reading of Veda summary 5):
over a short synthetic trajectory of layer inputs, the device's per-head
refresh decisions and ages equal the fp64 oracle's rule applied to the same
descriptors; a refreshed head's index lists equal a fresh score + top-k pass
bit for bit, and a reused head's equal the previous step's."""
import numpy as np
import pytest
import torch

import synth
from block_sparse_attention_24_b200.layer import VedaLayer, device_weights
from tests.helpers import small_workloads
from oracle import veda_oracle as O

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _layer(w, cache):
    import block_sparse_attention_24_b200 as V
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device=DEV)
    layer = VedaLayer(L, w.keep, device_weights(synth.mlp_weights(w), DEV), synth.SCORE_SCALE, DEV,
                      score_cache=cache)
    return V, L, layer


CASES = {"cfg0": lambda: synth.config(0), "cfg1": lambda: synth.config(1),
         "batch2": lambda: small_workloads()["batch2-d64-t128"],
         "padded-d128-t128": lambda: small_workloads()["ragged-d128-t128"]}


@pytest.mark.parametrize("name", list(CASES))
def test_score_cache_trajectory(name):
    w = CASES[name]()
    tau, max_age = 0.05, 3
    V, L, layer = _layer(w, (tau, max_age))
    q0, k0, v0 = synth.qkv(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    Hh = w.heads
    moved = [0, Hh - 1]                       # heads whose inputs change a lot on steps 1 and 3

    def perturbed(x, heads, sigma):
        y = x.clone()
        for h in heads:
            noise = torch.randn(y[:, :, h].shape, generator=g, device=DEV, dtype=torch.float32)
            y[:, :, h] = (y[:, :, h].float() + sigma * noise).to(y.dtype)
        return y

    # step inputs: 0 base; 1 large change on `moved`; 2 the same as 1; 3 large
    # change on `moved` again (the other heads reach max_age here)
    steps = [(q0, k0)]
    q1, k1 = perturbed(q0, moved, 2.0), perturbed(k0, moved, 2.0)
    steps += [(q1, k1), (q1, k1), (perturbed(q1, moved, 2.0), perturbed(k1, moved, 2.0))]

    nt = L.nt
    age = np.full(w.B * Hh, -1)
    ref_q = ref_k = np.zeros(tuple(layer.dq.shape))
    prev_idx = None
    fresh_scores = torch.empty_like(layer.scores)
    fresh_idx = torch.empty_like(layer.idx)
    wts = [layer.w[n] for n in ("w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k")]
    decisions = []
    for s, (q, k) in enumerate(steps):
        layer.front(q, k, v0)
        torch.cuda.synchronize()
        V.veda_check_status(L)
        dq, dk = layer.dq.cpu().double().numpy(), layer.dk.cpu().double().numpy()
        refresh, age, ref_q, ref_k = O.score_cache_step(dq, dk, ref_q, ref_k, nt, age, tau, max_age)
        assert layer.refresh.cpu().tolist() == refresh.tolist(), s
        assert layer.cache_age.cpu().tolist() == age.tolist(), s
        decisions.append(refresh.tolist())
        # a fresh score + top-k pass on this step's descriptors
        V.veda_tile_scores(L, layer.dq, layer.dk, *wts, layer.hidden, layer.out_dim, layer.score_scale,
                           fresh_scores, layer.emb_ws)
        V.veda_topk_mask(L, fresh_scores, layer.k, layer.k_cap, fresh_idx)
        torch.cuda.synchronize()
        for b in range(w.B):
            for h in range(Hh):
                got = layer.idx[b, h]
                if refresh[b * Hh + h]:
                    assert torch.equal(got, fresh_idx[b, h]), (s, h)
                else:
                    assert torch.equal(got, prev_idx[b, h]), (s, h)
        prev_idx = layer.idx.clone()
        # attention runs on the cached mask like on any other
        layer.attend()
        V.veda_check_status(L)
    ones, moved_only = [1] * (w.B * Hh), [int(h in moved) for h in range(Hh)] * w.B
    assert decisions[0] == ones                      # never scored
    assert decisions[1] == moved_only                # drift far above tau only there
    assert decisions[2] == [0] * (w.B * Hh)          # same inputs as step 1
    assert decisions[3] == ones                      # moved heads drift, the others reach max_age
