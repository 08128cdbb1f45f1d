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


def _tp_worker(rank, world, port, out):
    """Head-parallel ranks on CPU: each takes its head slice of the experts
    (api.head_slice), routes the same tokens with the replicated router and
    mixes only its rows (here with the oracle as the arithmetic); gathering
    the slices must give the unsharded result, with no collective needed in
    the value path itself."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import mova_inputs as MI
    from mixture_value_routing_b200.api import head_slice
    from oracle import mova_oracle as O

    dist.init_process_group("gloo")
    d, E, k, n, T = 128, 8, 2, 384, 6
    lay = MI.make_layer(3, 0, d=d, E=E, n=n, wv_dtype="f32")
    x = O.to_f64(MI.make_batch(T, 3, d=d, dtype="f32").x, "f32")  # the same tokens on every rank
    r = O.route(x, lay.Wr.astype(np.float64), lay.br.astype(np.float64), k, 2.5)
    row0, cnt = head_slice(n, world, rank)
    mine = O.combine(x, r["idx"], r["w"], lay.Wv[:, row0:row0 + cnt, :], "f32")
    sizes = [head_slice(n, world, q)[1] for q in range(world)]
    width = max(sizes)  # gloo gathers equal shapes: pad, then trim
    padded = torch.zeros((T, width), dtype=torch.float64)
    padded[:, :cnt] = torch.from_numpy(mine)
    gathered = [torch.zeros((T, width), dtype=torch.float64) for _ in sizes]
    dist.all_gather(gathered, padded)
    joined = torch.cat([g[:, :c] for g, c in zip(gathered, sizes)], dim=1).numpy()
    full = O.combine(x, r["idx"], r["w"], lay.Wv, "f32")
    out[rank] = (row0, cnt, float(np.abs(joined - full).max()))
    dist.destroy_process_group()


def test_two_rank_head_parallel_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_tp_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(out)
    assert res[0][:2] == (0, 256) and res[1][:2] == (256, 128)  # 3 heads: 2 + 1
    assert res[0][2] < 1e-12 and res[1][2] < 1e-12  # fp64 products of a slice vs the whole


def test_head_slice_deals_whole_heads():
    from mixture_value_routing_b200.api import head_slice
    for heads in (1, 3, 8):
        for world in range(1, heads + 1):
            got = [head_slice(heads * 128, world, r) for r in range(world)]
            assert got[0][0] == 0 and sum(c for _, c in got) == heads * 128
            for (a0, ac), (b0, _) in zip(got, got[1:]):
                assert a0 + ac == b0 and ac % 128 == 0 and ac > 0
