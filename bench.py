"""Benchmark of the Veda tile-skipping attention layer on B200.

A step is one pass of the whole hot path over one synthetic layer (the
720P-10s-like layer: 40x48x80 latent grid = 153,600 tokens, 24 heads, d=128,
128-token tiles, 10% of key tiles kept = 90% sparsity):
  permute Q,K,V -> TripPool Q,K -> MLP tile scores -> top-k mask
  -> tile-skipping sparse attention -> inverse permute
  -> full-attention tile map + row-wise KL on 2 heads x 120 query tiles
  -> recall of the top-k mask against the tile map's own top-k on those rows.

`value` is effective attention TFLOP/s over the whole step (4*d*kept valid
token pairs / step time); the attention kernel alone, the library's dense
path at sparsity 0 and the roofline of the attention kernel are reported
beside it. `--impl reference` times the fp64 CPU oracle on a bounded sample
of the same workload. Beside the step the line carries the same layer at 95%
sparsity (attention, dense-path speedup, recall) and the attention kernel on
the 24,576-token (64-token tiles) and 80,640-token layers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "block-sparse attn ms/layer & effective TFLOP/s at 90% sparsity vs dense path"
UNIT = "TFLOP/s"
MAP_ROWS = 120          # query tiles per tile-map head (10% of 1200: sparse supervision)
KERNELS_FRONT_ATTN = 7  # 2 permute+TripPool, permute V, MLP + score GEMM, top-k, attention (output in token order)
KERNELS_MAP = 6         # map sweep + finish, KL rows, KL mean, recall rows + mean


# ------------------------------------------------------------------ ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def dist_init(backend: str, world: int):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, device) -> float:
    """Largest value of x over all ranks (the timing rule: the job is as slow
    as its slowest rank)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device) -> float:
    """Sum of x over all ranks (host-side bookkeeping outside the timed region)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def rank_workload_seed(rank: int) -> int:
    """Each rank processes its own independent layer (weak scaling): same
    shapes, different seeded activations."""
    return 7919 * rank


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling (100 ms) of SM clock, power and throttle reasons.
    Started before the warm-up so its start-up never lands in the timed
    region; `summary(t0, t1)` keeps only samples taken inside [t0, t1]
    (host wall clock, as datetime.now())."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # raw samples go to $VEDA_CLOCKS_DIR (default: the system temp directory)
        self.path = os.path.join(os.environ.get("VEDA_CLOCKS_DIR") or tempfile.gettempdir(), f"clocks_rank{index}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self, t0=None, t1=None):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, pw, mx, reasons = [], [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f")
                clk, mx_, pwr = float(p[2]), float(p[3]), float(p[4])
            except ValueError:
                continue
            if t0 is not None and not (t0 <= ts <= t1):
                continue
            sm.append(clk)
            pw.append(pwr)
            mx = mx_
            for n, v in zip(names, p[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "power_w_median": statistics.median(pw) if pw else None, "samples": len(sm),
                "period_ms": 100}


def measured_clock_max():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    return json.load(open(p)).get("sm_max_mhz") if os.path.exists(p) else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d["bf16_tflops_sustained"], d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# --------------------------------------------------------------- our path

def layer_inputs(w, device, seed_offset=0, head_range=None):
    """Host-side description of the benchmark layer for workload w, or
    (head_range = (h0, h1)) of the same layer restricted to heads [h0, h1):
    (workload, scorer weights, (q, k, v), tile-map heads, their sampled query
    tiles). A restricted layer keeps those heads' tilings, weights, Q/K/V
    slices and tile-map rows, so a head computes exactly what it computes in
    the whole layer."""
    h0, h1 = (0, w.heads) if head_range is None else head_range
    sub = w if head_range is None else synth.head_subset(w, h0, h1)
    heads = list(sub.tilemap_heads)
    rows = None
    if heads:
        nts = [(sub.T + pt - 1) // pt * (sub.H // ph) * (sub.W // pw) for pt, ph, pw in sub.tilings]
        rows = np.stack([synth.sample_rows(nts[h], min(MAP_ROWS, nts[h]), w.seed + h0 + h) for h in heads])
    weights = tuple(a[h0:h1] for a in synth.mlp_weights(w))
    q, k, v = synth.qkv(w, device, seed_offset=seed_offset)
    if head_range is not None:
        q, k, v = (t[:, :, h0:h1].contiguous() for t in (q, k, v))
    return sub, weights, (q, k, v), heads, rows


def build_layer(w, device, seed_offset=0, head_range=None):
    """The benchmark layer (or its restriction to head_range) on the device."""
    import block_sparse_attention_24_b200 as V
    from block_sparse_attention_24_b200.layer import MapRequest, VedaLayer, device_weights
    sub, weights, (q, k, v), heads, rows = layer_inputs(w, device, seed_offset, head_range)
    L = V.Layer(sub.B, sub.heads, sub.d, sub.T, sub.H, sub.W, sub.tile, sub.tilings, device=device)
    maps = MapRequest(heads, torch.from_numpy(rows).to(device), rows.shape[1]) if heads else None
    layer = VedaLayer(L, w.keep, device_weights(weights, device), synth.SCORE_SCALE, device, maps=maps)
    return V, L, layer, (q, k, v)


def kept_pairs(L, layer, idx=None, k=None):
    """Kept valid (query, key) token pairs and all valid pairs, from the
    top-k lists (default: the layer's own) and the tile lengths."""
    idx = (layer.idx if idx is None else idx).cpu()
    k = layer.k if k is None else k
    kept = allp = 0
    for h in range(L.heads):
        pt, ph, pw = L.tilings[h]
        tps = (L.H // ph) * (L.W // pw)
        lens = torch.tensor([min(pt, L.T - (t // tps) * pt) * ph * pw for t in range(L.nt[h])], dtype=torch.int64)
        for b in range(L.B):
            rows = idx[b, h, :L.nt[h], :k[h]].long()
            kept += int((lens * lens[rows].sum(dim=1)).sum())
            allp += int(lens.sum()) ** 2
    return kept, allp


def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init("nccl", world)
    w = synth.config(args.config, keep=args.keep)
    head_range = None
    if args.shard_heads:
        # one layer, its heads split over the ranks (no exchange: every step is per head)
        from block_sparse_attention_24_b200.shard import head_ranges
        head_range = head_ranges(w.heads, world)[rank]
        if head_range[0] == head_range[1]:
            raise SystemExit(f"rank {rank}: no heads left for {world} ranks and {w.heads} heads")
        V, L, layer, (q, k, v) = build_layer(w, device, head_range=head_range)
    else:
        V, L, layer, (q, k, v) = build_layer(w, device, seed_offset=rank_workload_seed(rank))
    stream = torch.cuda.current_stream(device)

    clk = ClockSampler(local).__enter__()
    # warm-up
    for _ in range(args.warmup):
        layer.forward(q, k, v)
    torch.cuda.synchronize(device)
    V.veda_check_status(L)
    kept, allp = kept_pairs(L, layer)
    eff_flops = 4.0 * L.d * kept
    n_stage = len(layer.STAGES)

    # timed region: whole steps (layer.forward), with events at the stage
    # boundaries on the launching stream
    names = ("start", "front", "attn0", "attn1", "unpermute", "end")
    ev = [{n: torch.cuda.Event(enable_timing=True) for n in names} for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(device)
    if True:  # the timed region
        host_t0 = datetime.datetime.now()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(args.steps):
            layer.forward(q, k, v, marks=ev[s])
        t1.record(stream)
        torch.cuda.synchronize(device)
        host_t1 = datetime.datetime.now()
    barrier()
    elapsed = t0.elapsed_time(t1) / 1e3
    elapsed = max_over_ranks(elapsed, device)
    V.veda_check_status(L)
    front_ms = statistics.mean(e["start"].elapsed_time(e["front"]) for e in ev)
    attn_each = [e["attn0"].elapsed_time(e["attn1"]) for e in ev]
    attn_ms = statistics.mean(attn_each)  # the roofline's average launch duration
    unperm_ms = statistics.mean(e["attn1"].elapsed_time(e["unpermute"]) for e in ev)
    tail_ms = statistics.mean(e["unpermute"].elapsed_time(e["end"]) for e in ev)
    clk.__exit__(None, None, None)
    clocks = clk.summary(host_t0, host_t1)

    # per-stage breakdown of the front end (separate, untimed-for-value pass)
    stage_ms = stage_breakdown(V, L, layer, q, k, v, stream)
    grad_ms = estimator_grad_ms(layer, stream) if layer.maps is not None else None
    cache_ms = score_cache_ms(layer, q, k, v, stream)

    # dense path (same kernel, every tile kept) on the same permuted tensors
    dense_out = torch.empty_like(layer.op)
    layer.dense(dense_out)
    torch.cuda.synchronize(device)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = args.dense_reps
    d0.record(stream)
    for _ in range(reps):
        layer.dense(dense_out)
    d1.record(stream)
    torch.cuda.synchronize(device)
    dense_ms = d0.elapsed_time(d1) / reps
    del dense_out

    e2e = run_e2e(V, L, layer, q, k, v, device, eff_flops, args)

    burst, sustained, hbm, src = measured_peaks()
    attn_tflops = eff_flops / (attn_ms / 1e3) / 1e12
    layer_ms = front_ms + attn_ms + unperm_ms
    step_ms = elapsed / args.steps * 1e3
    total_flops = sum_over_ranks(eff_flops, device) if args.shard_heads else world * eff_flops
    value = total_flops / (elapsed / args.steps) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, layer, L, budget_s=args.cpu_seconds)
    traffic = load_traffic()
    hbm_stages = frontend_bandwidth(L, layer, stage_ms, unperm_ms, hbm)
    alu_stages = frontend_compute(L, layer, stage_ms, clocks.get("sm_mhz"))
    recall90 = layer_recall(layer) if layer.maps is not None else None
    map_rows = int(layer.maps.n_rows) if layer.maps is not None else MAP_ROWS
    map_kernels = layer.maps is not None
    sp95 = run_keep(V, L, layer, q, k, v, 0.05, dense_ms, burst, stream)
    del layer, q, k, v
    torch.cuda.empty_cache()
    others = {} if (args.no_other_layers or world > 1) else other_layers(device, burst, stream)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 3), "higher_is_better": True,
        "scaling": "strong" if args.shard_heads else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(w, world, round(1 - kept / allp, 4), map_rows, args.shard_heads),
        "attn_ms": round(attn_ms, 3), "attn_tflops": round(attn_tflops, 1),
        "attn_frac_of_burst_peak": round(attn_tflops / burst, 4),
        "attn_ms_median": round(statistics.median(attn_each), 3), "attn_ms_min": round(min(attn_each), 3),
        "dense_ms": round(dense_ms, 3), "speedup_vs_dense": round(dense_ms / attn_ms, 2),
        "layer_ms": round(layer_ms, 3),
        "speedup_layer_vs_dense": round(dense_ms / layer_ms, 2),
        "stage_ms": {**stage_ms, "front_end": round(front_ms, 3), "sparse_attn": round(attn_ms, 3),
                     "unpermute": round(unperm_ms, 3), "tilemap_kl": round(tail_ms, 3)},
        "estimator_grad_ms": grad_ms,
        "score_cache": cache_ms,
        "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 1), "peak": burst, "unit": UNIT,
                     "frac": round(attn_tflops / burst, 4), "traffic": traffic,
                     "kernel": "sparse_attn_pair_kernel<128>",
                     "kernel_source_sha256_16": kernel_source_hash(),
                     "peak_kind": f"bf16 dense burst ({src}): the kernel is timed launch by launch",
                     "frac_of_sustained": round(attn_tflops / sustained, 4)},
        "recall": recall90,
        "sparsity_95": sp95,
        "other_layers": others,
        "hbm_stages": hbm_stages,
        "alu_stages": alu_stages,
        "e2e": e2e,
        "gpu_launches": (KERNELS_FRONT_ATTN + (KERNELS_MAP if map_kernels else 0)) * args.steps,
        "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def layer_recall(layer) -> dict:
    """Recall of the step's top-k mask against the tile map's own top-k on
    the map rows (computed inside the step by the recall kernels)."""
    r = layer.recall.cpu().tolist()
    m = layer.maps
    return {"mean": round(r[-1], 4), "per_head": {str(h): round(x, 4) for h, x in zip(m.heads, r[:-1])},
            "rows_per_head": int(m.n_rows), "k": [layer.k[h] for h in m.heads],
            "note": "untrained (Xavier-initialised) estimator: reported, not targeted"}


def time_launches(fn, stream, reps, warm=2, flush=None):
    """Mean and min of `reps` launches of fn, each bracketed by CUDA events on
    `stream` (optionally writing `flush`, a buffer larger than L2, between
    launches)."""
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.add_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ts]
    return statistics.mean(ms), min(ms)


def run_keep(V, L, layer, q, k, v, keep, dense_ms, burst, stream, reps=10) -> dict:
    """The same layer at another keep fraction: top-k of the step's scores at
    that k, the attention kernel (output in token order) timed launch by
    launch, its speedup over the same dense-path time, and the recall of that
    mask against the step's tile map."""
    from block_sparse_attention_24_b200.layer import k_from_keep
    kk = [k_from_keep(keep, nt) for nt in L.nt]
    k_cap = max(kk)
    idx = torch.empty((L.B, L.heads, L.nt_cap, k_cap), dtype=torch.int32, device=layer.device)
    V.veda_topk_mask(L, layer.scores, kk, k_cap, idx, None)
    rec = None
    if layer.maps is not None:
        hits = torch.empty_like(layer.recall_hits)
        rec = torch.empty_like(layer.recall)
        layer.map_recall(idx, kk, k_cap, hits, rec)
    out = torch.empty_like(layer.o)
    fn = lambda: V.veda_sparse_attn_unpermute(L, layer.qp, layer.kp, layer.vp, idx, kk, k_cap, layer.attn_scale, out)
    mean_ms, min_ms = time_launches(fn, stream, reps)
    V.veda_check_status(L)
    kept, allp = kept_pairs(L, layer, idx, kk)
    tf = 4.0 * L.d * kept / (mean_ms / 1e3) / 1e12
    r = rec.cpu().tolist() if rec is not None else None
    return {"keep": keep, "k": kk[0] if len(set(kk)) == 1 else kk, "sparsity": round(1 - kept / allp, 4),
            "attn_ms": round(mean_ms, 3), "attn_ms_min": round(min_ms, 3), "attn_tflops": round(tf, 1),
            "attn_frac_of_burst_peak": round(tf / burst, 4), "speedup_vs_dense": round(dense_ms / mean_ms, 2),
            "recall": None if r is None else
            {"mean": round(r[-1], 4), "per_head": {str(h): round(x, 4) for h, x in zip(layer.maps.heads, r[:-1])}}}


def other_layers(device, burst, stream) -> dict:
    """The attention kernel on the 24,576-token layer (12 heads, 64-token
    tiles, 80% sparsity) and the 80,640-token layer (40 heads, T padded per
    tiling, 90% sparsity): each launch timed on its own after an L2 flush,
    and the same kernel's dense path."""
    out = {}
    flush = torch.empty(64 << 20, dtype=torch.float32, device=device)   # 256 MB > L2
    for cfg in (1, 2):
        w = synth.config(cfg)
        V, L, layer, (q, k, v) = build_layer(w, device)
        layer.forward(q, k, v)
        torch.cuda.synchronize()
        kept, allp = kept_pairs(L, layer)
        mean_ms, min_ms = time_launches(lambda: layer.attend(stream), stream, 10, flush=flush)
        dout = torch.empty_like(layer.op)
        dense_ms, _ = time_launches(lambda: layer.dense(dout), stream, 2, warm=1, flush=flush)
        V.veda_check_status(L)
        tf = 4.0 * L.d * kept / (mean_ms / 1e3) / 1e12
        out[w.name] = {"tokens": w.N, "heads": w.heads, "tile": w.tile, "sparsity": round(1 - kept / allp, 4),
                       "attn_ms": round(mean_ms, 3), "attn_ms_min": round(min_ms, 3), "attn_tflops": round(tf, 1),
                       "attn_frac_of_burst_peak": round(tf / burst, 4), "dense_ms": round(dense_ms, 3),
                       "dense_tflops": round(4.0 * L.d * allp / (dense_ms / 1e3) / 1e12, 1),
                       "speedup_vs_dense": round(dense_ms / mean_ms, 2), "l2": "flushed before every launch",
                       "recall": round(float(layer.recall[-1]), 4) if layer.maps is not None else None}
        del layer, q, k, v, dout
        torch.cuda.empty_cache()
    return out


def frontend_compute(L, layer, stage_ms, sm_mhz) -> dict:
    """The compute-bound front-end stages against bounds derived from the SM
    count and the sampled SM clock: the MLP and score GEMM against the fp32
    FMA rate (148 SMs x 128 FMA lanes x 2 flop per clock), the top-k against
    the instruction issue rate (148 SMs x 4 schedulers x 1 warp instruction
    per clock) for its counting loop (2 integer instructions per key and
    bisection step, 32 steps, keys padded to the register layout)."""
    clock_kind = "median SM clock sampled in the timed region"
    if not sm_mhz:   # no sample in a short timed region: the GPU's maximum clock
        sm_mhz = measured_clock_max()
        clock_kind = "maximum SM clock (no sample in the timed region)"
    if not sm_mhz:
        return {}
    f = sm_mhz * 1e6
    d3, hid, out_dim = 3 * L.d, layer.hidden, layer.out_dim
    nts = [L.nt[h] for h in range(L.heads)] * L.B
    mlp = sum(2 * nt * 2 * (d3 * hid + hid * out_dim) for nt in nts)
    gemm = sum(2 * nt * nt * out_dim for nt in nts)
    ffma_peak = 148 * 128 * 2 * f
    kpl = (L.nt_cap + 255) // 256 * 8
    rows = L.B * L.heads * L.nt_cap
    issue = rows * 32 * 2 * kpl
    issue_peak = 148 * 4 * f
    ts, tk = stage_ms["tile_scores"] / 1e3, stage_ms["topk"] / 1e3
    return {"clock_mhz": sm_mhz, "clock": clock_kind,
            "tile_scores": {"bound": "fp32 fma", "flop": mlp + gemm, "ms": stage_ms["tile_scores"],
                            "tflops": round((mlp + gemm) / ts / 1e12, 2), "peak_tflops": round(ffma_peak / 1e12, 1),
                            "frac": round((mlp + gemm) / ts / ffma_peak, 3)},
            "topk": {"bound": "issue", "warp_instructions": issue, "ms": stage_ms["topk"],
                     "frac": round(issue / tk / issue_peak, 3)}}


def stage_breakdown(V, L, layer, q, k, v, stream):
    names = ["permute_trippool_qk", "permute_v", "tile_scores", "topk"]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
    w = layer.w
    ev[0].record(stream)
    V.veda_permute_trippool(L, q, layer.qp, layer.dq, layer.perm)
    V.veda_permute_trippool(L, k, layer.kp, layer.dk)
    ev[1].record(stream)
    V.veda_permute(L, v, layer.vp)
    ev[2].record(stream)
    V.veda_tile_scores(L, layer.dq, layer.dk, w["w1q"], w["b1q"], w["w2q"], w["b2q"], w["w1k"], w["b1k"], w["w2k"],
                       w["b2k"], layer.hidden, layer.out_dim, layer.score_scale, layer.scores, layer.emb_ws)
    ev[3].record(stream)
    V.veda_topk_mask(L, layer.scores, layer.k, layer.k_cap, layer.idx, layer.mask)
    ev[4].record(stream)
    torch.cuda.synchronize()
    return {n: round(ev[i].elapsed_time(ev[i + 1]), 3) for i, n in enumerate(names)}


def score_cache_ms(layer, q, k, v, stream, reps=5):
    """Front end (Q/K permute + TripPool, V permute, then the scores and
    top-k) with temporal caching of tile scores: every head rebuilt (ages
    reset) vs every head reused (the same inputs again), plus the cache step
    alone. The benchmark's own step does not cache."""
    layer.enable_score_cache(0.05, 1 << 30)
    layer.front(q, k, v)

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ms = []
        for _ in range(reps):
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return round(statistics.median(ms), 3)

    def rebuilt():
        layer.cache_age.fill_(-1)
        layer.front(q, k, v)

    out = {"front_ms_rebuilt": timed(rebuilt), "front_ms_reused": timed(lambda: layer.front(q, k, v))}
    import block_sparse_attention_24_b200 as V
    out["cache_step_ms"] = timed(lambda: V.veda_score_cache_step(layer.L, layer.dq, layer.dk, layer.dq_ref, layer.dk_ref,
                                                                 0.05, 1 << 30, layer.cache_age, layer.refresh,
                                                                 layer.cache_ws))
    layer.score_cache = None
    return out


def estimator_grad_ms(layer, stream, reps=5):
    """One estimator-training gradient (the KL back through the score product
    and the MLP, on this step's tile-map rows): outside the step, reported
    beside it."""
    layer.estimator_grad()
    layer.estimator_grad()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        layer.estimator_grad()
    e1.record(stream)
    torch.cuda.synchronize()
    return round(e0.elapsed_time(e1) / reps, 3)


def run_e2e(V, L, layer, q, k, v, device, eff_flops, args):
    """Host buffers in, host result out, through the public pipelined call
    (HostPipeline): every step copies its Q, K, V from pinned host memory and
    its output and KL back, with the copies of neighbouring steps overlapping
    the kernels. The timed region starts before the first input copy and ends
    after the last output copy."""
    from block_sparse_attention_24_b200.layer import HostPipeline
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(layer.o.shape, dtype=layer.o.dtype).pin_memory()
    hkl = torch.empty(4, dtype=torch.float32).pin_memory()
    pipe = HostPipeline(layer, q)
    stream = torch.cuda.current_stream(device)
    pipe.run((hq, hk, hv), ho, hkl, steps=2)      # warm-up
    pipe.wait()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    pipe.run((hq, hk, hv), ho, hkl, steps=args.e2e_steps)
    pipe.wait()
    e1.record(stream)
    torch.cuda.synchronize(device)
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3 / args.e2e_steps, device)
    world = dist_env()[0]
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hkl.numel() * hkl.element_size()
    return {"value": round(world * eff_flops / t / 1e12, 3), "unit": UNIT, "ms_per_step": round(t * 1e3, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            "copies": "overlapped with the kernels of the neighbouring steps (two copy streams)"}


def bench_config(w, world, sparsity, map_rows, shard_heads=False) -> dict:
    """The workload description both arms print."""
    qkv_mb = w.B * w.N * w.heads * w.d * 2 / 1e6
    return {"workload": w.name, "model": "none (one attention layer, synthetic activations)",
            "global_batch": w.B * world, "seq_len": w.N, "heads": w.heads, "head_dim": w.d,
            "tile": w.tile, "keep": w.keep, "sparsity": sparsity,
            "tilemap": {"heads": list(w.tilemap_heads), "query_tiles_per_head": int(map_rows)},
            "parallelism": ("single GPU" if world == 1 else
                            f"one layer, heads split over {world} GPUs (no exchange)" if shard_heads else
                            "independent layer per GPU"),
            "l2": (f"inputs larger than L2 (each of Q/K/V is {qkv_mb:.0f} MB)" if qkv_mb > 126 else
                   f"inputs fit in L2 (each of Q/K/V is {qkv_mb:.0f} MB); parity-size layer, not the benchmark layer")}


def layout_sparsity(w) -> float:
    """Sparsity from the layout alone: exact when no head's T is padded (every
    tile full, so kept pairs = nt * k * tile^2 per head), else the nominal
    1 - keep."""
    kept = allp = 0
    for pt, ph, pw in w.tilings:
        if w.T % pt:
            return round(1 - w.keep, 4)
        nt = (w.T // pt) * (w.H // ph) * (w.W // pw)
        kk = max(1, int(math.floor(w.keep * nt + 0.5)))
        kept += nt * kk
        allp += nt * nt
    return round(1 - kept / allp, 4)


def kernel_source_hash() -> str:
    """Hash of the attention kernel's device source: attn_pair.cu, walk.cuh
    and the device-code part of veda_internal.cuh (its host launcher
    declarations at the end change with unrelated entry points)."""
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_attention_24_b200", "csrc")
    hsh = hashlib.sha256()
    hsh.update(open(os.path.join(csrc, "attn_pair.cu"), "rb").read())
    hsh.update(open(os.path.join(csrc, "walk.cuh"), "rb").read())
    hdr = open(os.path.join(csrc, "veda_internal.cuh"), "rb").read()
    hsh.update(hdr.split(b"// Host-side launchers")[0])
    return hsh.hexdigest()[:16]


def load_traffic():
    """DRAM bytes (read + write) per attention launch at this workload, from
    the committed ncu summary; None once the kernel source differs from the
    one the counters were taken on."""
    p = os.path.join(ROOT, "profiles", "sparse_attn_traffic_153600tok.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if d.get("kernel_source_sha256_16") == kernel_source_hash():
            return d.get("dram_bytes_per_launch")
    return None


def frontend_bandwidth(L, layer, stage_ms, unperm_ms, hbm_gbs):
    """Algorithmic HBM bytes of the bandwidth-bound stages and the achieved
    rate against the measured HBM copy bandwidth."""
    Hh, d, B = L.heads, L.d, L.B
    valid = sum(L.N for _ in range(Hh)) * B          # valid token rows over heads
    row = d * 2
    nt_sum = sum(L.nt) * B
    byts = {
        # Q and K: read every original row, write every permuted row (incl.
        # padding) and [avg|max|min] fp32 per tile
        "permute_trippool_qk": 2 * (valid * row + B * Hh * L.n_cap * row + nt_sum * 3 * d * 4),
        # V: read every original row, write every permuted row
        "permute_v": valid * row + B * Hh * L.n_cap * row,
        # read the scores, write index lists and the dense mask
        "topk": B * Hh * L.nt_cap * L.nt_cap * 4 + B * Hh * L.nt_cap * (layer.k_cap * 4 + L.nt_cap),

    }
    out = {}
    for k, b in byts.items():
        ms = stage_ms[k]
        out[k] = {"bytes": b, "ms": ms, "gbs": round(b / (ms / 1e3) / 1e9, 1),
                  "frac_of_measured_hbm": round(b / (ms / 1e3) / 1e9 / hbm_gbs, 3)}
    # the inverse permutation is the attention kernel's output store: no
    # separate pass, its 2 x 0.94 GB of traffic is gone
    out["unpermute"] = {"fused": "the attention epilogue writes each output row to its token", "ms": unperm_ms}
    return out


# ------------------------------------------------------------ CPU oracle

def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_attention_sample(w, qp_h, kp_h, vp_h, idx_h, k, lens, budget_s, seed=0):
    """Runs the oracle's sparse attention tile by tile on seeded query tiles
    until `budget_s` seconds are used; returns (effective flops, seconds,
    tiles)."""
    from oracle import veda_oracle as O
    nt = len(lens)
    order = np.random.default_rng(seed).permutation(nt)
    flops, tiles = 0.0, 0
    t0 = time.perf_counter()
    for a in order:
        O.sparse_attention(qp_h, kp_h, vp_h, idx_h, k, lens, w.tile, 1 / math.sqrt(w.d), rows=[int(a)])
        flops += 4.0 * w.d * O.effective_pairs(lens, idx_h, k, rows=[int(a)])
        tiles += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return flops, time.perf_counter() - t0, tiles


def cpu_baseline(w, layer, L, budget_s):
    from oracle import veda_oracle as O
    h = 0
    lens = O.head_layout(w.T, w.H, w.W, w.tilings[h])["lens"]
    f = lambda t: t[0, h].float().cpu().double().numpy()
    torch.cuda.synchronize()    # the layer permutes V on its side stream
    qp, kp, vp = f(layer.qp), f(layer.kp), f(layer.vp)
    idx = layer.idx[0, h].cpu().numpy()
    flops, secs, tiles = oracle_attention_sample(w, qp, kp, vp, idx, layer.k[h], lens, budget_s)
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"fp64 NumPy sparse attention, head {h}, {tiles} random query tiles of {L.nt[h]} "
                      f"({secs:.1f} s); the front end is not included"}


def run_reference(args, world, rank, local):
    """The fp64 CPU oracle as the reference arm: each step = the oracle's
    front end for one head (permute, TripPool, MLP scores, top-k) plus its
    sparse attention on seeded query tiles of that head."""
    if rank != 0:
        return
    from oracle import veda_oracle as O
    w = synth.config(args.config, keep=args.keep)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    q, k, v = synth.qkv(w, dev)
    w1, b1, w2, b2 = synth.mlp_weights(w)
    h = 0
    tiling = w.tilings[h]
    lay = O.head_layout(w.T, w.H, w.W, tiling)
    perm = O.perm_indices(w.T, w.H, w.W, tiling)
    qh, kh, vh = (t[:, :, h:h + 1].float().cpu().double().numpy() for t in (q, k, v))
    del q, k, v
    kk = O.k_from_keep(w.keep, lay["nt"])

    def step(budget):
        t0 = time.perf_counter()
        qp, kp, vp = (O.permute(x, [perm], lay["n_pad"])[0, 0] for x in (qh, kh, vh))
        dq = O.trippool(qp, lay["lens"], w.tile)
        dk = O.trippool(kp, lay["lens"], w.tile)
        s = O.tile_scores(dq, dk, w1[h], b1[h], w2[h], b2[h], w1[h], b1[h], w2[h], b2[h], synth.SCORE_SCALE)
        idx, _ = O.topk_rows(s, kk)
        front = time.perf_counter() - t0
        flops, secs, tiles = oracle_attention_sample(w, qp, kp, vp, idx, kk, lay["lens"], budget)
        return flops, front + secs, tiles

    for _ in range(args.warmup):
        step(1.0)
    tot_f = tot_s = 0.0
    tiles = 0
    for _ in range(args.steps):
        f, s_, t = step(args.ref_step_seconds)
        tot_f += f
        tot_s += s_
        tiles += t
    value = tot_f / tot_s / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(tot_s / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": bench_config(w, world, layout_sparsity(w), MAP_ROWS),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"per step: oracle front end for head {h} + sparse attention on "
                                   f"~{tiles / max(1, args.steps):.0f} seeded query tiles"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """Head-group sweep (8 heads, d=128, 128-token tiles): sparse attention at
    each keep fraction against the same kernel's dense path, per token count.
    Prints one JSON object per point (not the benchmark contract line)."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    burst, sustained, _, src = measured_peaks()
    out = []
    for tokens in synth.SWEEP_TOKENS:
        dense_ms = None
        for keep in sorted(synth.SWEEP_KEEP, reverse=True):
            w = synth.sweep(tokens, keep)
            V, L, layer, (q, k, v) = build_layer(w, device)
            layer.front(q, k, v)
            torch.cuda.synchronize()
            kept, allp = kept_pairs(L, layer)
            flops = 4.0 * L.d * kept
            args_attn = (L, layer.qp, layer.kp, layer.vp, layer.idx, layer.k, layer.k_cap, layer.attn_scale, layer.op)
            for _ in range(2):
                V.veda_sparse_attn(*args_attn)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            e0.record()
            for _ in range(reps):
                V.veda_sparse_attn(*args_attn)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            if dense_ms is None:
                dout = torch.empty_like(layer.op)
                layer.dense(dout)
                e0.record()
                for _ in range(3):
                    layer.dense(dout)
                e1.record()
                torch.cuda.synchronize()
                dense_ms = e0.elapsed_time(e1) / 3
                dense_flops = 4.0 * L.d * allp
                del dout
            V.veda_check_status(L)
            rec = {"tokens": w.N, "keep": keep, "sparsity": round(1 - kept / allp, 4), "k": layer.k[0],
                   "attn_ms": round(ms, 3), "eff_tflops": round(flops / ms / 1e9, 1),
                   "frac_of_burst_peak": round(flops / ms / 1e9 / burst, 4), "dense_ms": round(dense_ms, 3),
                   "dense_tflops": round(dense_flops / dense_ms / 1e9, 1), "speedup_vs_dense": round(dense_ms / ms, 2)}
            print(json.dumps(rec), flush=True)
            out.append(rec)
            del layer, q, k, v
            torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--keep", type=float, default=None)
    ap.add_argument("--dense-reps", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=24)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-layers", action="store_true", help="skip the 24,576- and 80,640-token attention timings")
    ap.add_argument("--sweep", action="store_true", help="head-group token/sparsity sweep instead of the step")
    ap.add_argument("--shard-heads", action="store_true",
                    help="N>1: one layer with its heads split over the ranks (strong scaling) instead of an "
                         "independent layer per rank")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps are required")
    world, rank, local = dist_env()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
