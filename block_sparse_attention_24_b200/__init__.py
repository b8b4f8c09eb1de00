"""Python binding of libveda.so, the B200 (sm_100a) hot path of Veda's
distilled tile-skipping sparse attention ("Technical Summary: Veda - Scalable
Video Diffusion via Distilled Sparse Attention", sections 2.1-2.3).

Argument marshalling only: every function here passes device pointers and
sizes to the C ABI declared in include/veda.h, on the current torch CUDA
stream. There is no CPU or PyTorch fallback; if the library is missing the
import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libveda.so")

VEDA_OK = 0
VEDA_ERR_INVALID_ARG = -1
VEDA_ERR_UNSUPPORTED = -2
VEDA_ERR_CUDA = -3
VEDA_ERR_TIMEOUT = -4
VEDA_ERR_BAD_INDEX = -5

EXPORTED = ("veda_layout", "veda_permute", "veda_trippool", "veda_permute_trippool", "veda_tile_scores", "veda_tile_scores_ws_bytes",
            "veda_tile_scores_noalloc",
            "veda_topk_mask", "veda_tile_scores_topk", "veda_tile_scores_heads", "veda_topk_mask_heads", "veda_score_cache_step", "veda_score_cache_ws_bytes", "veda_sparse_attn", "veda_sparse_attn_unpermute", "veda_sparse_attn_tokens", "veda_full_attn_tilemax", "veda_full_attn_tilemax_ws_bytes", "veda_tilemap_kl", "veda_tilemap_recall",
            "veda_check_status",
            "veda_estimator_grad", "veda_estimator_grad_ws_bytes", "veda_output_sq_error", "veda_selftest_wait_timeout", "veda_last_error")


class VedaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"veda error {code}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python block_sparse_attention_24_b200/build.py`")
    return ctypes.CDLL(_LIB_PATH)


_lib = _load()


class _Tiling(ctypes.Structure):
    _fields_ = [("pt", ctypes.c_int32), ("ph", ctypes.c_int32), ("pw", ctypes.c_int32)]


class _Layer(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("d", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("tile", ctypes.c_int32),
                ("tilings", ctypes.POINTER(_Tiling)), ("dev_status", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_LP = ctypes.POINTER(_Layer)
_lib.veda_layout.argtypes = [_LP, _P, _P, _P, _P]
_lib.veda_permute.argtypes = [_LP, _P, _P, _P, ctypes.c_int, _P]
_lib.veda_trippool.argtypes = [_LP, _P, _P, _P]
_lib.veda_permute_trippool.argtypes = [_LP, _P, _P, _P, _P, _P]
_lib.veda_tile_scores.argtypes = [_LP] + [_P] * 10 + [_I, _I, _F, _P, _P, _P]
_lib.veda_tile_scores_noalloc.argtypes = [_LP] + [_P] * 10 + [_I, _I, _F, _P, _P]
_lib.veda_tile_scores_ws_bytes.argtypes = [_LP, _I]
_lib.veda_tile_scores_ws_bytes.restype = ctypes.c_size_t
_lib.veda_topk_mask.argtypes = [_LP, _P, _P, _I, _P, _P, _P]
_lib.veda_tile_scores_heads.argtypes = [_LP] + [_P] * 10 + [_I, _I, _F, _P, _P, _P, _P]
_lib.veda_topk_mask_heads.argtypes = [_LP, _P, _P, _I, _P, _P, _P, _P]
_lib.veda_score_cache_step.argtypes = [_LP, _P, _P, _P, _P, _F, _I, _P, _P, _P, _P]
_lib.veda_score_cache_ws_bytes.argtypes = [_LP]
_lib.veda_score_cache_ws_bytes.restype = ctypes.c_size_t
_lib.veda_tile_scores_topk.argtypes = [_LP] + [_P] * 10 + [_I, _I, _F, _P, _I, _P, _P, _P, _P, _P]
_lib.veda_sparse_attn.argtypes = [_LP, _P, _P, _P, _P, _P, _I, _F, _P, _P, _P]
_lib.veda_sparse_attn_unpermute.argtypes = [_LP, _P, _P, _P, _P, _P, _I, _F, _P, _P, _P]
_lib.veda_sparse_attn_tokens.argtypes = [_LP, _P, _P, _P, _P, _P, _I, _F, _P, _P, _P]
_lib.veda_full_attn_tilemax.argtypes = [_LP, _P, _P, _P, _I, _P, _I, _F, _P, _P, _P, _P, _P, _P, _P]
_lib.veda_full_attn_tilemax_ws_bytes.argtypes = [_LP, _I, _I]
_lib.veda_tilemap_kl.argtypes = [_LP, _P, _I, _P, _I, _P, _P, _P, _P, _P]
_lib.veda_full_attn_tilemax_ws_bytes.restype = ctypes.c_size_t
_lib.veda_tilemap_recall.argtypes = [_LP, _P, _I, _P, _I, _P, _P, _P, _I, _P, _P, _P, _P]
_lib.veda_estimator_grad.argtypes = [_LP] + [_P] * 10 + [_I, _I, _F, _P, _I, _P, _I, _P] + [_P] * 8 + [_P, _P, _P]
_lib.veda_estimator_grad_ws_bytes.argtypes = [_LP, _I, _I, _I, _I]
_lib.veda_estimator_grad_ws_bytes.restype = ctypes.c_size_t
_lib.veda_output_sq_error.argtypes = [_LP, _P, _P, _P, _P]
_lib.veda_check_status.argtypes = [_LP, _P]
_lib.veda_selftest_wait_timeout.argtypes = [_LP, ctypes.c_uint32, _P]
_lib.veda_last_error.restype = ctypes.c_char_p
for _name in EXPORTED:
    getattr(_lib, _name)
    if _name not in ("veda_last_error", "veda_tile_scores_ws_bytes", "veda_estimator_grad_ws_bytes",
                     "veda_full_attn_tilemax_ws_bytes", "veda_score_cache_ws_bytes"):
        getattr(_lib, _name).restype = ctypes.c_int


def veda_last_error() -> str:
    return _lib.veda_last_error().decode()


def _check(rc: int):
    if rc != VEDA_OK:
        raise VedaError(rc, veda_last_error())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libveda must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Layer:
    """Geometry of one attention layer (veda_layer) plus its device status
    word. `tilings` is one (p_t, p_h, p_w) per head."""

    def __init__(self, B: int, heads: int, d: int, T: int, H: int, W: int, tile: int,
                 tilings: Sequence[Tuple[int, int, int]], device=None):
        self.B, self.heads, self.d, self.T, self.H, self.W, self.tile = B, heads, d, T, H, W, tile
        self.tilings = [tuple(int(v) for v in t) for t in tilings]
        self._til = (_Tiling * max(1, heads))(*[_Tiling(*t) for t in self.tilings])
        self.status = None
        if device is not None:
            self.status = torch.zeros(4, dtype=torch.int32, device=device)
        self._c = _Layer(B, heads, d, T, H, W, tile, ctypes.cast(self._til, ctypes.POINTER(_Tiling)),
                         ctypes.c_void_p(self.status.data_ptr()) if self.status is not None else None)
        nt = (ctypes.c_int32 * max(1, heads))()
        npad = (ctypes.c_int32 * max(1, heads))()
        ncap, ntcap = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.veda_layout(ctypes.byref(self._c), nt, npad, ctypes.byref(ncap), ctypes.byref(ntcap)))
        self.nt = list(nt)[:heads]
        self.n_pad = list(npad)[:heads]
        self.n_cap = ncap.value
        self.nt_cap = ntcap.value

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def ref(self):
        return ctypes.byref(self._c)


def veda_layout(layer: Layer):
    """(nt per head, n_pad per head, n_cap, nt_cap)."""
    return layer.nt, layer.n_pad, layer.n_cap, layer.nt_cap


def veda_permute(layer: Layer, x: torch.Tensor, xp: torch.Tensor, perm: Optional[torch.Tensor] = None,
                 inverse: bool = False, stream=None):
    _check(_lib.veda_permute(layer.ref, _ptr(x), _ptr(xp), _ptr(perm), int(inverse), _stream(stream)))


def veda_trippool(layer: Layer, xp: torch.Tensor, desc: torch.Tensor, stream=None):
    _check(_lib.veda_trippool(layer.ref, _ptr(xp), _ptr(desc), _stream(stream)))


def veda_permute_trippool(layer: Layer, x: torch.Tensor, xp: torch.Tensor, desc: torch.Tensor,
                          perm: Optional[torch.Tensor] = None, stream=None):
    _check(_lib.veda_permute_trippool(layer.ref, _ptr(x), _ptr(xp), _ptr(perm), _ptr(desc), _stream(stream)))


def veda_tile_scores_ws_bytes(layer: Layer, out_dim: int) -> int:
    return int(_lib.veda_tile_scores_ws_bytes(layer.ref, out_dim))


def veda_tile_scores(layer: Layer, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden: int, out_dim: int,
                     scale: float, scores: torch.Tensor, emb_ws: torch.Tensor, stream=None):
    _check(_lib.veda_tile_scores(layer.ref, *[_ptr(t) for t in (dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k)],
                                 hidden, out_dim, float(scale), _ptr(scores), _ptr(emb_ws), _stream(stream)))


def veda_tile_scores_noalloc(layer: Layer, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden: int,
                             out_dim: int, scale: float, scores: torch.Tensor, stream=None):
    """veda_tile_scores for callers that cannot allocate device memory: the
    embeddings go to a 16 MiB array built into the library (shared by all
    calls; overlapping calls race)."""
    _check(_lib.veda_tile_scores_noalloc(layer.ref, *[_ptr(t) for t in (dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k,
                                                                         b2k)],
                                         hidden, out_dim, float(scale), _ptr(scores), _stream(stream)))


def _host_i32(vals):
    arr = (ctypes.c_int32 * max(1, len(vals)))(*[int(v) for v in vals])
    return arr


def veda_topk_mask(layer: Layer, scores: torch.Tensor, k: Sequence[int], k_cap: int, idx: torch.Tensor,
                   mask: Optional[torch.Tensor] = None, stream=None):
    _check(_lib.veda_topk_mask(layer.ref, _ptr(scores), _host_i32(k), int(k_cap), _ptr(idx), _ptr(mask),
                               _stream(stream)))


def veda_tile_scores_heads(layer: Layer, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden: int,
                           out_dim: int, scale: float, scores: torch.Tensor, emb_ws: torch.Tensor,
                           head_on: Optional[torch.Tensor], stream=None):
    """veda_tile_scores for the (batch element, head) pairs with head_on != 0."""
    _check(_lib.veda_tile_scores_heads(layer.ref, *[_ptr(t) for t in (dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k,
                                                                        b2k)],
                                       hidden, out_dim, float(scale), _ptr(scores), _ptr(emb_ws), _ptr(head_on),
                                       _stream(stream)))


def veda_topk_mask_heads(layer: Layer, scores: torch.Tensor, k: Sequence[int], k_cap: int, idx: torch.Tensor,
                         mask: Optional[torch.Tensor], head_on: Optional[torch.Tensor], stream=None):
    """veda_topk_mask for the (batch element, head) pairs with head_on != 0."""
    _check(_lib.veda_topk_mask_heads(layer.ref, _ptr(scores), _host_i32(k), int(k_cap), _ptr(idx), _ptr(mask),
                                     _ptr(head_on), _stream(stream)))


def veda_score_cache_ws_bytes(layer: Layer) -> int:
    return int(_lib.veda_score_cache_ws_bytes(layer.ref))


def veda_score_cache_step(layer: Layer, dq, dk, dq_ref, dk_ref, tau: float, max_age: int, age: torch.Tensor,
                          refresh: torch.Tensor, ws: torch.Tensor, stream=None):
    """Temporal caching of tile scores: per (batch element, head), decide on
    the device whether its cached mask is reused (refresh 0) or rebuilt."""
    _check(_lib.veda_score_cache_step(layer.ref, _ptr(dq), _ptr(dk), _ptr(dq_ref), _ptr(dk_ref), float(tau),
                                      int(max_age), _ptr(age), _ptr(refresh), _ptr(ws), _stream(stream)))


def veda_tile_scores_topk(layer: Layer, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden: int, out_dim: int,
                          scale: float, k: Sequence[int], k_cap: int, idx: torch.Tensor, emb_ws: torch.Tensor,
                          mask: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None, stream=None):
    _check(_lib.veda_tile_scores_topk(layer.ref, *[_ptr(t) for t in (dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k)],
                                      hidden, out_dim, float(scale), _host_i32(k), int(k_cap), _ptr(idx), _ptr(mask),
                                      _ptr(scores), _ptr(emb_ws), _stream(stream)))


def veda_sparse_attn(layer: Layer, qp, kp, vp, idx: Optional[torch.Tensor], k: Optional[Sequence[int]], k_cap: int,
                     scale: float, op: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    karr = _host_i32(k) if k is not None else None
    _check(_lib.veda_sparse_attn(layer.ref, _ptr(qp), _ptr(kp), _ptr(vp), _ptr(idx), karr, int(k_cap),
                                 float(scale), _ptr(op), _ptr(lse), _stream(stream)))


def veda_sparse_attn_unpermute(layer: Layer, qp, kp, vp, idx: Optional[torch.Tensor], k: Optional[Sequence[int]],
                               k_cap: int, scale: float, o: torch.Tensor, lse: Optional[torch.Tensor] = None,
                               stream=None):
    """veda_sparse_attn with the output written in token order [B, N, heads, d]."""
    karr = _host_i32(k) if k is not None else None
    _check(_lib.veda_sparse_attn_unpermute(layer.ref, _ptr(qp), _ptr(kp), _ptr(vp), _ptr(idx), karr, int(k_cap),
                                           float(scale), _ptr(o), _ptr(lse), _stream(stream)))


def veda_sparse_attn_tokens(layer: Layer, q, k, v, idx: Optional[torch.Tensor], kk: Optional[Sequence[int]],
                            k_cap: int, scale: float, o: torch.Tensor, lse: Optional[torch.Tensor] = None,
                            stream=None):
    """Sparse attention with q, k, v and o in token order [B, N, heads, d]."""
    karr = _host_i32(kk) if kk is not None else None
    _check(_lib.veda_sparse_attn_tokens(layer.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), karr, int(k_cap),
                                        float(scale), _ptr(o), _ptr(lse), _stream(stream)))


def veda_full_attn_tilemax(layer: Layer, qp, kp, heads_sel: Sequence[int], qtile_rows: Optional[torch.Tensor],
                           n_rows: int, scale: float, tilemap: torch.Tensor, lse: Optional[torch.Tensor] = None,
                           scores: Optional[torch.Tensor] = None, kl_rows: Optional[torch.Tensor] = None,
                           kl_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    _check(_lib.veda_full_attn_tilemax(layer.ref, _ptr(qp), _ptr(kp), _host_i32(heads_sel), len(heads_sel),
                                       _ptr(qtile_rows), int(n_rows), float(scale), _ptr(tilemap), _ptr(lse),
                                       _ptr(scores), _ptr(kl_rows), _ptr(kl_out), _ptr(ws), _stream(stream)))


def veda_tilemap_kl(layer: Layer, heads_sel: Sequence[int], qtile_rows: Optional[torch.Tensor], n_rows: int,
                    tilemap: torch.Tensor, scores: torch.Tensor, kl_rows: torch.Tensor, kl_out: torch.Tensor,
                    stream=None):
    _check(_lib.veda_tilemap_kl(layer.ref, _host_i32(heads_sel), len(heads_sel), _ptr(qtile_rows), int(n_rows),
                                _ptr(tilemap), _ptr(scores), _ptr(kl_rows), _ptr(kl_out), _stream(stream)))


def veda_tilemap_recall(layer: Layer, heads_sel: Sequence[int], qtile_rows: Optional[torch.Tensor], n_rows: int,
                        tilemap: torch.Tensor, idx: torch.Tensor, k: Sequence[int], k_cap: int, hits: torch.Tensor,
                        recall: torch.Tensor, map_idx: Optional[torch.Tensor] = None, stream=None):
    """hits [n_heads_sel, n_rows] int32, recall [n_heads_sel + 1] fp32 (per
    head, then their mean); map_idx (optional) the map's own top-k lists."""
    _check(_lib.veda_tilemap_recall(layer.ref, _host_i32(heads_sel), len(heads_sel), _ptr(qtile_rows), int(n_rows),
                                    _ptr(tilemap), _ptr(idx), _host_i32(k), int(k_cap), _ptr(hits), _ptr(map_idx),
                                    _ptr(recall), _stream(stream)))


def veda_full_attn_tilemax_ws_bytes(layer: Layer, n_heads_sel: int, n_rows: int) -> int:
    return int(_lib.veda_full_attn_tilemax_ws_bytes(layer.ref, n_heads_sel, n_rows))


def veda_estimator_grad_ws_bytes(layer: Layer, n_heads_sel: int, n_rows: int, hidden: int, out_dim: int) -> int:
    return int(_lib.veda_estimator_grad_ws_bytes(layer.ref, n_heads_sel, n_rows, hidden, out_dim))


def veda_estimator_grad(layer: Layer, dq, dk, weights: Sequence[torch.Tensor], hidden: int, out_dim: int,
                        scale: float, heads_sel: Sequence[int], qtile_rows: Optional[torch.Tensor], n_rows: int,
                        tilemap: torch.Tensor, grads: Sequence[torch.Tensor], ws: torch.Tensor,
                        loss: Optional[torch.Tensor] = None, stream=None):
    """weights and grads: (w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k)."""
    _check(_lib.veda_estimator_grad(layer.ref, _ptr(dq), _ptr(dk), *[_ptr(t) for t in weights], hidden, out_dim,
                                    float(scale), _host_i32(heads_sel), len(heads_sel), _ptr(qtile_rows),
                                    int(n_rows), _ptr(tilemap), *[_ptr(t) for t in grads], _ptr(loss), _ptr(ws),
                                    _stream(stream)))


def veda_output_sq_error(layer: Layer, a: torch.Tensor, b: torch.Tensor, err: torch.Tensor, stream=None):
    _check(_lib.veda_output_sq_error(layer.ref, _ptr(a), _ptr(b), _ptr(err), _stream(stream)))


def veda_check_status(layer: Layer, stream=None):
    _check(_lib.veda_check_status(layer.ref, _stream(stream)))


def veda_selftest_wait_timeout(layer: Layer, limit_ms: int, stream=None):
    _check(_lib.veda_selftest_wait_timeout(layer.ref, int(limit_ms), _stream(stream)))


def library_path() -> str:
    return _LIB_PATH
