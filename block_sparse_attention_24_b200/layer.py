"""One Veda attention layer on the device: the C-ABI calls of the hot path in
order, over buffers allocated once.

    permute + TripPool (Q, K), permute (V) -> tile scores -> top-k mask
      -> tile-skipping sparse attention -> inverse permute
    (+ distillation rows: full-attention tile map on selected heads and query
       tiles, row-wise KL against the predicted scores, recall of the
       predicted mask against the map's own top-k)

Only marshalling and buffer management live here; every step is a libveda
kernel launch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import (Layer, veda_estimator_grad, veda_estimator_grad_ws_bytes, veda_full_attn_tilemax,
               veda_full_attn_tilemax_ws_bytes, veda_permute, veda_permute_trippool, veda_sparse_attn,
               veda_sparse_attn_unpermute, veda_score_cache_step, veda_score_cache_ws_bytes, veda_tile_scores,
               veda_tile_scores_heads, veda_tilemap_recall,
               veda_topk_mask_heads,
               veda_tile_scores_ws_bytes, veda_topk_mask)


def k_from_keep(keep: float, nt: int) -> int:
    """Kept key tiles per query tile: round-half-up of keep*nt, at least 1."""
    return max(1, int(math.floor(keep * nt + 0.5)))


@dataclass
class MapRequest:
    heads: List[int]                 # heads whose tile map is built
    rows: Optional[torch.Tensor]     # device int32 [len(heads), n_rows] or None (tiles 0..n_rows-1)
    n_rows: int


class VedaLayer:
    STAGES = ("permute_trippool_q", "permute_trippool_k", "permute_v", "tile_scores", "topk", "sparse_attn",
              "unpermute", "tilemap_kl")

    def __init__(self, layer: Layer, keep: Optional[float], weights: Dict[str, torch.Tensor], score_scale: float,
                 device, k: Optional[Sequence[int]] = None, maps: Optional[MapRequest] = None,
                 score_cache: Optional[Tuple[float, int]] = None):
        """score_cache: (tau, max_age) to reuse each head's tile scores and
        top-k mask across steps while its descriptors drift less than tau
        (veda_score_cache_step); None rebuilds them every step."""
        self.L = layer
        self.device = device
        B, Hh, d = layer.B, layer.heads, layer.d
        self.k = list(k) if k is not None else [k_from_keep(keep, nt) for nt in layer.nt]
        self.k_cap = max(self.k)
        self.hidden = int(weights["w1q"].shape[-1])
        self.out_dim = int(weights["w2q"].shape[-1])
        self.w = weights
        self.score_scale = float(score_scale)
        self.attn_scale = 1.0 / math.sqrt(d)
        n_cap, nt_cap = layer.n_cap, layer.nt_cap
        bf = dict(dtype=torch.bfloat16, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.qp = torch.empty((B, Hh, n_cap, d), **bf)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty_like(self.qp)
        self.op = torch.empty_like(self.qp)
        self.dq = torch.empty((B, Hh, nt_cap, 3 * d), **f32)
        self.dk = torch.empty_like(self.dq)
        self.scores = torch.empty((B, Hh, nt_cap, nt_cap), **f32)
        self.emb_ws = torch.empty(veda_tile_scores_ws_bytes(layer, self.out_dim) // 4, **f32)
        self.idx = torch.empty((B, Hh, nt_cap, self.k_cap), dtype=torch.int32, device=device)
        self.mask = torch.empty((B, Hh, nt_cap, nt_cap), dtype=torch.uint8, device=device)
        self.perm = torch.empty((Hh, n_cap), dtype=torch.int32, device=device)
        self.o = torch.empty((B, layer.N, Hh, d), **bf)
        self.score_cache = None
        if score_cache is not None:
            self.enable_score_cache(*score_cache)
        self.maps = maps
        if maps is not None:
            nh = len(maps.heads)
            self.tilemap = torch.empty((nh, maps.n_rows, nt_cap), **f32)
            self.map_lse = torch.empty((nh, maps.n_rows, layer.tile), **f32)
            self.kl_rows = torch.empty((nh, maps.n_rows), **f32)
            self.kl_out = torch.zeros(4, **f32)
            self.map_ws = torch.empty(veda_full_attn_tilemax_ws_bytes(layer, nh, maps.n_rows) // 4, **f32)
            self.recall_hits = torch.empty((nh, maps.n_rows), dtype=torch.int32, device=device)
            self.recall = torch.zeros(nh + 1, **f32)   # per map head, then their mean

    def enable_score_cache(self, tau: float, max_age: int):
        """Start caching tile scores across steps (every head is rebuilt on
        the next step); disable with `self.score_cache = None`."""
        self.score_cache = (float(tau), int(max_age))
        if not hasattr(self, "dq_ref"):
            n = self.L.B * self.L.heads
            self.dq_ref = torch.zeros_like(self.dq)
            self.dk_ref = torch.zeros_like(self.dk)
            self.cache_age = torch.full((n,), -1, dtype=torch.int32, device=self.device)
            self.refresh = torch.ones((n,), dtype=torch.int32, device=self.device)
            nbytes = veda_score_cache_ws_bytes(self.L)
            self.cache_ws = torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device=self.device)
        self.cache_age.fill_(-1)

    def effective_flops(self, idx_host=None) -> float:
        """4*d*sum of kept valid (query, key) token pairs over all heads, from
        the tile lengths (host arithmetic on the layout)."""
        L = self.L
        total = 0
        for h in range(L.heads):
            pt, ph, pw = L.tilings[h]
            nt = L.nt[h]
            tps = (L.H // ph) * (L.W // pw)
            lens = [min(pt, L.T - (t // tps) * pt) * ph * pw for t in range(nt)]
            if idx_host is None:
                # every query tile keeps k tiles; exact count needs the lists
                raise ValueError("pass the index lists")
            for b in range(L.B):
                rows = idx_host[b, h, :nt, : self.k[h]]
                key_tok = torch.tensor(lens, dtype=torch.int64)[rows.long()].sum(dim=1)
                total += int((torch.tensor(lens, dtype=torch.int64) * key_tok).sum())
        return 4.0 * L.d * total

    # -- the hot path -------------------------------------------------------
    def front(self, q, k, v, stream=None):
        L = self.L
        # Q and K: permutation and TripPool in one pass; V: permutation only
        veda_permute_trippool(L, q, self.qp, self.dq, self.perm, stream=stream)
        veda_permute_trippool(L, k, self.kp, self.dk, stream=stream)
        veda_permute(L, v, self.vp, stream=stream)
        w = self.w
        wts = (w["w1q"], w["b1q"], w["w2q"], w["b2q"], w["w1k"], w["b1k"], w["w2k"], w["b2k"])
        if self.score_cache is None:
            veda_tile_scores(L, self.dq, self.dk, *wts, self.hidden, self.out_dim, self.score_scale, self.scores,
                             self.emb_ws, stream=stream)
            veda_topk_mask(L, self.scores, self.k, self.k_cap, self.idx, self.mask, stream=stream)
        else:
            # per head on the device: reuse the cached scores and mask, or rebuild them
            tau, max_age = self.score_cache
            veda_score_cache_step(L, self.dq, self.dk, self.dq_ref, self.dk_ref, tau, max_age, self.cache_age,
                                  self.refresh, self.cache_ws, stream=stream)
            veda_tile_scores_heads(L, self.dq, self.dk, *wts, self.hidden, self.out_dim, self.score_scale,
                                   self.scores, self.emb_ws, self.refresh, stream=stream)
            veda_topk_mask_heads(L, self.scores, self.k, self.k_cap, self.idx, self.mask, self.refresh,
                                 stream=stream)

    def attend(self, stream=None, out: Optional[torch.Tensor] = None):
        """Sparse attention with the output written in token order into `out`
        (default: the layer's own output buffer): one kernel, the inverse
        permutation fused into its epilogue."""
        veda_sparse_attn_unpermute(self.L, self.qp, self.kp, self.vp, self.idx, self.k, self.k_cap, self.attn_scale,
                                   self.o if out is None else out, stream=stream)

    def attend_permuted(self, stream=None):
        """Sparse attention into the permuted buffer `op` (one row per tile
        slot, padding rows zero), as the separate inverse permutation reads it."""
        veda_sparse_attn(self.L, self.qp, self.kp, self.vp, self.idx, self.k, self.k_cap, self.attn_scale, self.op,
                         stream=stream)

    def distill(self, stream=None):
        if self.maps is None:
            return
        m = self.maps
        veda_full_attn_tilemax(self.L, self.qp, self.kp, m.heads, m.rows, m.n_rows, self.attn_scale, self.tilemap,
                               self.map_lse, self.scores, self.kl_rows, self.kl_out, ws=self.map_ws, stream=stream)
        self.map_recall(self.idx, self.k, self.k_cap, self.recall_hits, self.recall, stream=stream)

    def map_recall(self, idx, k, k_cap, hits, recall, map_idx=None, stream=None):
        """Recall of predicted key-tile lists `idx` (k per head) against the
        top-k of this step's tile-map rows (call after distill's map)."""
        m = self.maps
        veda_tilemap_recall(self.L, m.heads, m.rows, m.n_rows, self.tilemap, idx, k, k_cap, hits, recall,
                            map_idx=map_idx, stream=stream)

    def estimator_grad(self, stream=None):
        """Weight gradient of the distillation loss on this step's tile-map
        rows (call after distill()): returns the eight gradient arrays
        (w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k) and the loss, on the device.
        The layer ties one MLP to both sides, so its gradient is the sum of
        the query and key parts."""
        m = self.maps
        if m is None:
            raise ValueError("estimator_grad needs tile-map rows (maps=...)")
        names = ("w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k")
        if not hasattr(self, "_grads"):
            self._grads = [torch.empty_like(self.w[n]) for n in names]
            self._grad_loss = torch.empty(1, dtype=torch.float32, device=self.device)
            nbytes = veda_estimator_grad_ws_bytes(self.L, len(m.heads), m.n_rows, self.hidden, self.out_dim)
            self._grad_ws = torch.empty(nbytes // 4, dtype=torch.float32, device=self.device)
        veda_estimator_grad(self.L, self.dq, self.dk, [self.w[n] for n in names], self.hidden, self.out_dim,
                            self.score_scale, m.heads, m.rows, m.n_rows, self.tilemap, self._grads, self._grad_ws,
                            self._grad_loss, stream=stream)
        return self._grads, self._grad_loss

    def forward(self, q, k, v, stream=None, out: Optional[torch.Tensor] = None, marks=None):
        """One step of the hot path, in order on one stream. `marks` (optional
        dict of CUDA events) is recorded at the stage boundaries "start",
        "front", "attn0", "attn1", "unpermute", "end" (the inverse permutation
        is fused into attention, so "attn1" and "unpermute" coincide). (Running the tile map
        on a second stream beside the rest measured slower: the split map
        already fills every SM.)"""
        main = torch.cuda.current_stream(self.device) if stream is None else stream

        def mark(name):
            if marks is not None and name in marks:
                marks[name].record(main)

        mark("start")
        self.front(q, k, v, main)
        mark("front")
        mark("attn0")
        self.attend(main, out)      # the inverse permutation is the attention epilogue's store
        mark("attn1")
        mark("unpermute")
        self.distill(main)
        mark("end")
        return self.o if out is None else out

    def dense(self, out: torch.Tensor, stream=None):
        """Same kernel with every tile kept (the library's own dense path)."""
        veda_sparse_attn(self.L, self.qp, self.kp, self.vp, None, None, 0, self.attn_scale, out, stream=stream)


def device_weights(np_weights, device) -> Dict[str, torch.Tensor]:
    """The same per-head MLP for query and key descriptors (w1, b1, w2, b2)."""
    w1, b1, w2, b2 = (torch.from_numpy(a).to(device) for a in np_weights)
    return {"w1q": w1, "b1q": b1, "w2q": w2, "b2q": b2, "w1k": w1, "b1k": b1, "w2k": w2, "b2k": b2}


class HostPipeline:
    """Runs a layer over host-resident inputs with the copies hidden behind
    the kernels: while step i computes, the host->device copy of step i+1's
    Q, K, V and the device->host copy of step i-1's output run on two copy
    streams (PCIe moves both directions at once). Two device input sets and
    two device output buffers alternate; events order every reuse. Each step
    still copies its own inputs in and its own output (and KL) out."""

    def __init__(self, layer: VedaLayer, q_like: torch.Tensor):
        dev = layer.device
        self.layer = layer
        self.inputs = [[torch.empty_like(q_like, device=dev) for _ in range(3)] for _ in range(2)]
        self.outputs = [torch.empty_like(layer.o) for _ in range(2)]
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.compute_done = [None, None]   # compute of the step that last used slot s
        self.d2h_done = [None, None]       # output copy of the step that last used slot s

    def run(self, host_qkv, host_out, host_kl=None, steps: int = 1):
        """host_qkv: pinned (q, k, v) host tensors; host_out: pinned host
        tensor of the output's shape (and host_kl of kl_out's, optional),
        rewritten every step. Returns when every copy has been enqueued."""
        comp = torch.cuda.current_stream(self.layer.device)
        for i in range(steps):
            s = i % 2
            dq, dk, dv = self.inputs[s]
            if self.compute_done[s] is not None:
                self.h2d.wait_event(self.compute_done[s])     # slot s's inputs are free again
            with torch.cuda.stream(self.h2d):
                for dst, src in zip((dq, dk, dv), host_qkv):
                    dst.copy_(src, non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(self.h2d)
            comp.wait_event(loaded)
            if self.d2h_done[s] is not None:
                comp.wait_event(self.d2h_done[s])             # slot s's output was copied out
            layer = self.layer
            layer.forward(dq, dk, dv, out=self.outputs[s])
            if host_kl is not None and layer.maps is not None:
                host_kl.copy_(layer.kl_out, non_blocking=True)
            done = torch.cuda.Event()
            done.record(comp)
            self.compute_done[s] = done
            self.d2h.wait_event(done)
            with torch.cuda.stream(self.d2h):
                host_out.copy_(self.outputs[s], non_blocking=True)
                copied = torch.cuda.Event()
                copied.record(self.d2h)
            self.d2h_done[s] = copied

    def wait(self):
        """Make the current stream wait for every copy issued so far."""
        comp = torch.cuda.current_stream(self.layer.device)
        for e in self.d2h_done:
            if e is not None:
                comp.wait_event(e)
