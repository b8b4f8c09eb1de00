"""Head-aware tiling search on the GPU (calibrate.choose_tilings, built from
the library's own calls) against the oracle's tiling_errors: the designed
frame / column locality case picks the designed tilings, and on synthetic
activations each candidate's per-head error matches the oracle within the
bf16 output noise."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_24_b200 as V
from block_sparse_attention_24_b200.calibrate import choose_tilings, tiling_errors
import synth
from oracle import veda_oracle as O

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def test_designed_locality_picks_designed_tilings():
    """Head 0 attends within its frame (one-hot of t), head 1 within its pair
    of x columns over all frames (one-hot of x // 2): whole-frame tiles
    (1,8,8) and column-pair tiles (4,8,2) are the right tilings."""
    T, H, W, d, tile = 4, 8, 8, 64, 64
    N = T * H * W
    t, y, x = (a.ravel() for a in np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij"))
    q = np.zeros((1, N, 2, d), np.float32)
    q[0, np.arange(N), 0, t] = 12.0
    q[0, np.arange(N), 1, x // 2] = 12.0
    v = np.random.default_rng(4).standard_normal((1, N, 2, d)).astype(np.float32)
    qb, vb = (torch.from_numpy(a).bfloat16().to(DEV) for a in (q, v))
    cands = [(1, 8, 8), (4, 8, 2)]
    choice, err = choose_tilings(qb, qb, vb, T, H, W, tile, cands, 0.25)
    assert choice == [(1, 8, 8), (4, 8, 2)]
    ref = O.tiling_errors(q, q, vb.double().cpu().numpy(), T, H, W, cands, 0.25, 1 / math.sqrt(d))
    assert list(np.argmin(ref, axis=0)) == [0, 1]
    e = err.numpy()
    assert e[0, 0] < 1e-2 * e[1, 0] and e[1, 1] < 1e-2 * e[0, 1]


@pytest.mark.parametrize("name,cands", [
    ("tile128", [(1, 8, 16), (2, 8, 8), (4, 4, 8)]),
    ("tile64", [(1, 8, 8), (4, 4, 4), (2, 4, 8)]),
])
def test_errors_match_oracle_on_synthetic_activations(name, cands):
    if name == "tile128":
        w = synth.custom("cal128", 1, 3, 128, 4, 8, 16, 128, [(1, 8, 16)] * 3, 0.25, 41)
    else:
        w = synth.custom("cal64", 1, 3, 64, 4, 8, 8, 64, [(1, 8, 8)] * 3, 0.25, 42)
    q, k, v = synth.qkv(w, "cpu")
    err = tiling_errors(q.to(DEV), k.to(DEV), v.to(DEV), w.T, w.H, w.W, w.tile, cands, w.keep).numpy()
    ref = O.tiling_errors(q.double().numpy(), k.double().numpy(), v.double().numpy(), w.T, w.H, w.W, cands,
                          w.keep, 1 / math.sqrt(w.d))
    # Each error is sum (d + e)^2 over the head's outputs, d = O_full - O_sparse
    # and e the GPU's error in d. Both outputs are bf16 within the attention
    # tolerance (|O| ~ 1), so e has rms at most 2^-8 and sum e^2 <= F below;
    # Cauchy-Schwarz then bounds |gpu - oracle| = |2 sum d e + sum e^2| by
    # 2 sqrt(oracle * F) + F.
    floor = w.N * w.d * (2.0 ** -8) ** 2
    assert np.all(np.abs(err - ref) <= 2 * np.sqrt(ref * floor) + floor), (err, ref, floor)
    for h in range(w.heads):     # the choice agrees wherever the oracle's margin is clear
        order = np.argsort(ref[:, h])
        if ref[order[1], h] > 1.2 * ref[order[0], h] + floor:
            assert np.argmin(err[:, h]) == order[0]


def test_output_sq_error_kernel():
    w = synth.custom("e", 2, 3, 128, 2, 8, 16, 128, [(1, 8, 16)] * 3, 1.0, 43)
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device=DEV)
    g = torch.Generator().manual_seed(5)
    a = torch.randn((w.B, w.N, w.heads, w.d), generator=g).bfloat16()
    b = torch.randn((w.B, w.N, w.heads, w.d), generator=g).bfloat16()
    err = torch.empty(4, dtype=torch.float32, device=DEV)
    V.veda_output_sq_error(L, a.to(DEV), b.to(DEV), err)
    ref = ((a.double() - b.double()) ** 2).sum(dim=(0, 1, 3)).numpy()
    np.testing.assert_allclose(err[:w.heads].cpu().numpy(), ref, rtol=1e-5)
