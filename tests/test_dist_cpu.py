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
