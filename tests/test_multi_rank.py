"""The multi-process (N > 1) host logic of bench.py on CPU with gloo, world
size 2: rank seeding (own tokens, shared weights), the max-over-ranks timing
reduction and the whole-job throughput.  The value path itself has no
collective: ranks process independent batches (weak scaling)."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    import mova_inputs as MI

    r, local, w = bench.dist_env()
    assert (r, local, w) == (rank, rank, world)
    on = bench.init_dist(w, "gloo")
    assert on and dist.get_world_size() == world
    bench.barrier(on)
    ms = bench.allmax(10.0 + 5.0 * rank, on, "cpu")
    x = MI.make_batch(16, bench.rank_batch_seed(0, rank), step=0, d=128).x
    lay = MI.make_layer(0, 0, d=128, E=4, n=128)
    xs = torch.tensor([float(x.astype(np.float64).sum())], dtype=torch.float64)
    ws = torch.tensor([float(lay.Wr.astype(np.float64).sum())], dtype=torch.float64)
    gx = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    gw = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(gx, xs)
    dist.all_gather(gw, ws)
    out[rank] = (ms, bench.job_value(w, 8, 100, ms), [float(t) for t in gx], [float(t) for t in gw])
    dist.destroy_process_group()


def test_two_rank_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(out)
    for rank in range(world):
        ms, value, gx, gw = res[rank]
        assert ms == 15.0  # the slowest rank's time, on every rank
        assert abs(value - 2 * 8 * 100 / 0.015) < 1e-6
        assert gx[0] != gx[1]  # own tokens per rank
        assert gw[0] == gw[1]  # the same layer weights on every rank
