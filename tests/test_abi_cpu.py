"""C-ABI checks that need no GPU: the library loads, exports every function
include/veda.h declares, computes layouts on the host and rejects bad
arguments before touching CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_24_b200 as V
import synth
from oracle import veda_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "veda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(veda_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert "veda_sparse_attn" in names and len(names) >= 10
    lib = ctypes.CDLL(V.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(V.EXPORTED)


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_layout_matches_oracle(idx):
    w = synth.config(idx)
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings)
    lays = [O.head_layout(w.T, w.H, w.W, t) for t in w.tilings]
    assert L.nt == [l["nt"] for l in lays]
    assert L.n_pad == [l["n_pad"] for l in lays]
    assert L.n_cap == max(l["n_pad"] for l in lays)
    assert L.nt_cap == max(l["nt"] for l in lays)


def test_sweep_layouts_have_no_padding():
    for n in synth.SWEEP_TOKENS:
        w = synth.sweep(n, 0.1)
        L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings)
        assert all(p == w.N for p in L.n_pad)


@pytest.mark.parametrize("tilings,msg", [
    ([(2, 8, 4)], "factorise"),
    ([(1, 8, 16)], "divide"),     # W=8 not divisible by 16
    ([(0, 8, 16)], "non-positive"),
])
def test_bad_tilings_rejected(tilings, msg):
    with pytest.raises(V.VedaError) as e:
        V.Layer(1, 1, 128, 4, 8, 8, 128, tilings)
    assert e.value.code == V.VEDA_ERR_INVALID_ARG and msg in str(e.value)


def test_unsupported_sizes_rejected():
    with pytest.raises(V.VedaError) as e:
        V.Layer(1, 1, 96, 4, 8, 8, 128, [(2, 8, 8)])
    assert e.value.code == V.VEDA_ERR_UNSUPPORTED
    with pytest.raises(V.VedaError) as e:
        V.Layer(1, 1, 128, 4, 8, 8, 32, [(1, 4, 8)])
    assert e.value.code == V.VEDA_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected_before_launch():
    L = V.Layer(1, 2, 64, 4, 8, 8, 64, [(1, 8, 8), (4, 4, 4)])
    lib = V._lib
    rc = lib.veda_permute(L.ref, None, None, None, 0, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "NULL" in V.veda_last_error()
    rc = lib.veda_permute(L.ref, ctypes.c_void_p(0x1008), ctypes.c_void_p(0x2000), None, 0, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "aligned" in V.veda_last_error()
    rc = lib.veda_permute_trippool(L.ref, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), None, None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "desc" in V.veda_last_error()
    rc = lib.veda_permute_trippool(L.ref, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3004),
                                   ctypes.c_void_p(0x4000), None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "perm" in V.veda_last_error()
    k = (ctypes.c_int32 * 2)(5, 1)      # k > nt for head 0
    rc = lib.veda_topk_mask(L.ref, ctypes.c_void_p(0x1000), k, 8, ctypes.c_void_p(0x2000), None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "k=5" in V.veda_last_error()
    rc = lib.veda_sparse_attn(L.ref, *[ctypes.c_void_p(0x1000)] * 3, None, None, 0, ctypes.c_float(-1.0),
                              ctypes.c_void_p(0x1000), None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "scale" in V.veda_last_error()
    rc = lib.veda_sparse_attn_unpermute(L.ref, *[ctypes.c_void_p(0x1000)] * 3, None, None, 0, ctypes.c_float(0.1),
                                        None, None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "o is NULL" in V.veda_last_error()
    rc = lib.veda_sparse_attn_unpermute(L.ref, *[ctypes.c_void_p(0x1000)] * 3, None, None, 0, ctypes.c_float(0.1),
                                        ctypes.c_void_p(0x1008), None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "aligned" in V.veda_last_error()
    rc = lib.veda_sparse_attn_tokens(L.ref, ctypes.c_void_p(0x1004), *[ctypes.c_void_p(0x1000)] * 2, None, None, 0,
                                     ctypes.c_float(0.1), ctypes.c_void_p(0x2000), None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "q is not 16-byte aligned" in V.veda_last_error()
    Q = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(7)]
    rc = lib.veda_score_cache_step(L.ref, *Q[:4], ctypes.c_float(-0.1), 3, Q[4], Q[5], Q[6], None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "tau" in V.veda_last_error()
    rc = lib.veda_score_cache_step(L.ref, *Q[:4], ctypes.c_float(0.1), 0, Q[4], Q[5], Q[6], None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "max_age" in V.veda_last_error()
    P = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(10)]
    rc = lib.veda_tile_scores_topk(L.ref, *P, 128, 64, ctypes.c_float(0.125), None, 4, ctypes.c_void_p(0x20000), None,
                                   None, ctypes.c_void_p(0x30000), None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "k is NULL" in V.veda_last_error()
    rc = lib.veda_tile_scores_topk(L.ref, *P, 102, 64, ctypes.c_float(0.125), k, 8, ctypes.c_void_p(0x20000), None,
                                   None, ctypes.c_void_p(0x30000), None)
    assert rc == V.VEDA_ERR_UNSUPPORTED and "hidden" in V.veda_last_error()
    rc = lib.veda_tile_scores_topk(L.ref, *P, 128, 64, ctypes.c_float(0.125), k, 8, None, None, None,
                                   ctypes.c_void_p(0x30000), None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "idx" in V.veda_last_error()
    sel = (ctypes.c_int32 * 1)(7)
    rc = lib.veda_full_attn_tilemax(L.ref, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), sel, 1, None, 1,
                                    ctypes.c_float(0.1), ctypes.c_void_p(0x1000), None, None, None, None, None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "heads_sel" in V.veda_last_error()
    rc = lib.veda_tilemap_kl(L.ref, sel, 1, None, 1, ctypes.c_void_p(0x1000), None, None, None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "scores" in V.veda_last_error()
    k_ok = (ctypes.c_int32 * 2)(2, 1)
    rc = lib.veda_tilemap_recall(L.ref, sel, 1, None, 1, *[ctypes.c_void_p(0x1000)] * 2, k_ok, 8,
                                 *[ctypes.c_void_p(0x1000)] * 3, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "heads_sel" in V.veda_last_error()
    sel0 = (ctypes.c_int32 * 1)(0)
    rc = lib.veda_tilemap_recall(L.ref, sel0, 1, None, 1, *[ctypes.c_void_p(0x1000)] * 2, k, 8,
                                 *[ctypes.c_void_p(0x1000)] * 3, None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "k=5" in V.veda_last_error()
    rc = lib.veda_tilemap_recall(L.ref, sel0, 1, None, 1, *[ctypes.c_void_p(0x1000)] * 2, k_ok, 8,
                                 None, None, ctypes.c_void_p(0x1000), None)
    assert rc == V.VEDA_ERR_INVALID_ARG and "hits" in V.veda_last_error()
    rc = lib.veda_check_status(None, None)
    assert rc == V.VEDA_ERR_INVALID_ARG


def test_tile_scores_workspace_size():
    w = synth.config(3)
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings)
    assert V.veda_tile_scores_ws_bytes(L, 64) == 2 * 24 * 1200 * 64 * 4


def test_empty_and_oversized_layers_rejected():
    with pytest.raises(V.VedaError) as e:
        V.Layer(1, 1, 128, 0, 8, 8, 128, [(2, 8, 8)])
    assert e.value.code == V.VEDA_ERR_INVALID_ARG and "empty" in str(e.value)
    with pytest.raises(V.VedaError) as e:
        V.Layer(0, 1, 128, 4, 8, 8, 128, [(2, 8, 8)])
    assert e.value.code == V.VEDA_ERR_INVALID_ARG
    with pytest.raises(V.VedaError) as e:      # 8200 tiles of 64 tokens > the 8192-tile limit
        V.Layer(1, 1, 128, 8200, 8, 8, 64, [(1, 8, 8)])
    assert e.value.code == V.VEDA_ERR_UNSUPPORTED and "exceeds" in str(e.value)
    with pytest.raises(V.VedaError):
        V.Layer(1, 129, 128, 4, 8, 8, 128, [(2, 8, 8)] * 129)


def test_token_attention_tiling_limit():
    """The token-order attention path keeps one tensor map per distinct tiling
    and takes at most 8 of them: a layer with 9 is refused on the host,
    before anything reaches the device."""
    tilings = [(1, 8, 16), (1, 16, 8), (2, 8, 8), (2, 4, 16), (2, 16, 4), (4, 4, 8), (4, 8, 4), (8, 4, 4),
               (8, 2, 8)]
    L = V.Layer(1, len(tilings), 64, 16, 16, 16, 128, tilings)
    lib = ctypes.CDLL(V.library_path())
    p = ctypes.c_void_p(0x10000)
    rc = lib.veda_sparse_attn_tokens(L.ref, p, p, p, None, None, 0, ctypes.c_float(0.125), p, None, None)
    assert rc == V.VEDA_ERR_UNSUPPORTED and "8 distinct tilings" in V.veda_last_error()
