"""The benchmark's multi-rank logic on CPU ranks (gloo, world size 2): each
rank gets its own layer (weak scaling, no data-path collective) and the step
time is the maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import synth
    w_, r_, l_ = bench.dist_env()
    bench.dist_init("gloo", w_)
    t = bench.max_over_ranks(1.5 + r_, "cpu")
    bench.barrier()
    tiny = synth.config(0)
    q, _, _ = synth.qkv(tiny, "cpu", seed_offset=bench.rank_workload_seed(r_))
    out[rank] = (w_, r_, t, float(q.float().sum()))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        w_, r_, t, _ = out[r]
        assert (w_, r_) == (world, r)
        assert t == pytest.approx(2.5)       # max over ranks of 1.5 + rank
    assert out[0][3] != out[1][3]            # independent layers per rank


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import numpy as np
    import bench
    import synth
    import torch
    from block_sparse_attention_24_b200.shard import head_ranges, local_heads
    w_, r_, _ = bench.dist_env()
    bench.dist_init("gloo", w_)
    full = synth.config(1)                     # 12 heads, 24,576 tokens, two tile-map heads
    h0, h1 = head_ranges(full.heads, w_)[r_]
    # the rank's share as bench.py --shard-heads builds it, against the whole layer's
    sub, wts, (q, k, v), mh, rows = bench.layer_inputs(full, "cpu", head_range=(h0, h1))
    fsub, fwts, (fq, fk, fv), fmh, frows = bench.layer_inputs(full, "cpu")
    ok_tilings = sub.tilings == full.tilings[h0:h1] and sub.heads == h1 - h0
    ok_weights = all(np.array_equal(a, b[h0:h1]) for a, b in zip(wts, fwts))
    ok_q = all(torch.equal(x, y[:, :, h0:h1]) for x, y in ((q, fq), (k, fk), (v, fv)))
    ok_maps = mh == local_heads(fmh, h0, h1) and all(
        np.array_equal(rows[i], frows[fmh.index(h0 + h)]) for i, h in enumerate(mh))
    gathered = [None] * w_
    torch.distributed.all_gather_object(gathered, (h0, h1))
    heads_done = bench.sum_over_ranks(h1 - h0, "cpu")
    out[rank] = (gathered, ok_tilings, ok_weights, ok_q, ok_maps, heads_done, [h0 + h for h in mh])
    torch.distributed.destroy_process_group()


def test_head_shards_cover_every_head_once():
    """bench.py --shard-heads: the ranks' head blocks partition the layer's
    heads, and each rank's tilings, scorer weights, Q/K/V, tile-map heads and
    their sampled query tiles are the whole layer's for those heads."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    blocks = out[0][0]
    assert blocks == out[1][0]
    covered = [h for h0, h1 in blocks for h in range(h0, h1)]
    assert covered == list(range(12))          # every head exactly once, in order
    map_heads = []
    for r in range(world):
        _, ok_t, ok_w, ok_q, ok_m, heads_done, mh = out[r]
        assert ok_t and ok_w and ok_q and ok_m
        assert heads_done == 12
        map_heads += mh
    import synth
    assert sorted(map_heads) == sorted(synth.config(1).tilemap_heads)


def test_head_ranges_balanced():
    from block_sparse_attention_24_b200.shard import head_ranges, local_heads
    for n, world in [(24, 1), (24, 5), (24, 8), (40, 3), (3, 4)]:
        r = head_ranges(n, world)
        assert len(r) == world and r[0][0] == 0 and r[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        sizes = [h1 - h0 for h0, h1 in r]
        assert max(sizes) - min(sizes) <= 1
    assert local_heads([3, 7, 12], 5, 13) == [2, 7]
