"""The allocation-free tile-score call (veda_tile_scores_noalloc) against the
regular one (veda_tile_scores with a caller scratch buffer).

Some callers cannot allocate device memory at all: plug-in hosts that own a
pre-planned device memory pool, and real-time loops that must not enter an
allocator between frames. For them the library keeps the embedding scratch in
a built-in device array. This checks, through the C ABI, that two calls in a
row (the second with different inputs, so stale scratch contents would show)
give the regular call's scores bit for bit (both run the same kernels on the
same inputs), that a call after the first one changes no device memory
reservation, and that a layer too large for the built-in array is refused.
It lives in its own file so that it runs last."""
import numpy as np
import pytest
import torch

import block_sparse_attention_24_b200 as V
import synth

pytestmark = pytest.mark.gpu


def _inputs(w, nt_cap, seed):
    rng = np.random.default_rng(seed)
    dq = rng.standard_normal((w.B, w.heads, nt_cap, 3 * w.d)).astype(np.float32)
    dk = rng.standard_normal((w.B, w.heads, nt_cap, 3 * w.d)).astype(np.float32)
    w1, b1, w2, b2 = synth.mlp_weights(w)
    b1 = (rng.standard_normal(b1.shape) * 0.1).astype(np.float32)
    b2 = (rng.standard_normal(b2.shape) * 0.1).astype(np.float32)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return [T(a) for a in (dq, dk, w1, b1, w2, b2, w1 * 0.5, b1, w2, b2)]


def test_noalloc_matches_regular_call_twice():
    w = synth.config(1)                      # 12 heads x 384 tiles, d=128, tile 64
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device="cuda")
    shape = (w.B, w.heads, L.nt_cap, L.nt_cap)
    ws = torch.empty(V.veda_tile_scores_ws_bytes(L, synth.MLP_OUT) // 4, dtype=torch.float32, device="cuda")
    for seed in (1, 2):                      # two calls in a row through the shared scratch
        args = _inputs(w, L.nt_cap, seed)
        want = torch.empty(shape, dtype=torch.float32, device="cuda")
        got = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        V.veda_tile_scores(L, *args, synth.MLP_HIDDEN, synth.MLP_OUT, synth.SCORE_SCALE, want, ws)
        V.veda_tile_scores_noalloc(L, *args, synth.MLP_HIDDEN, synth.MLP_OUT, synth.SCORE_SCALE, got)
        V.veda_check_status(L)
        assert torch.isfinite(got).all()
        assert torch.equal(got, want)
    # the first call on this device has set up its scratch address; later
    # calls reserve no device memory
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    V.veda_tile_scores_noalloc(L, *args, synth.MLP_HIDDEN, synth.MLP_OUT, synth.SCORE_SCALE, got)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.equal(got, want)


def test_noalloc_refuses_layers_beyond_its_scratch():
    # 48 heads x 1200 tiles x 64 outputs x 2 sides x 4 bytes = 29.5 MB > 16 MiB
    L = V.Layer(1, 48, 128, 40, 48, 80, 128, [(2, 8, 8)] * 48, device="cuda")
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(V.VedaError) as e:
        V.veda_tile_scores_noalloc(L, *([dummy] * 10), synth.MLP_HIDDEN, synth.MLP_OUT, synth.SCORE_SCALE, dummy)
    assert e.value.code == V.VEDA_ERR_UNSUPPORTED and "scratch" in str(e.value)
