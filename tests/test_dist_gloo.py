"""The multi-process logic of bench.py on CPU: two gloo ranks.

Each rank scans its own independent copy of the workload (different seeds, no
exchange on the data path), the timings are reduced with a maximum over ranks,
and the whole-job rate counts every rank's elements over the slowest rank's
time.  The data path itself is also shown to shard without exchange: two ranks
running the fp64 oracle on disjoint channel halves reproduce the one-process
result exactly once gathered.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from selective_state_space_36_b200 import inputs as I
        cfg = bench.rank_config(rank)
        first = I.draw_rows(cfg, "u", 0, 0, 4)
        got = [None] * world
        dist.all_gather_object(got, first.tobytes())
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank])
        rate = bench.whole_job_rate(world, 1000, mx[0])
        # shard a small problem by channels: rank r takes half of the dims
        small = I.ScanConfig("shard", 2, 40, 12, 4, io="bf16", seed=3, h0_sigma=0.2)
        x = I.scan_inputs(small)
        lo, hi = rank * small.dim // world, (rank + 1) * small.dim // world
        f = lambda k: I.to_f64(x[k], "bf16")
        sl = slice(lo, hi)
        o, st = oracle.scan(f("u")[:, :, sl], f("delta")[:, :, sl], x["A"][sl].astype(float), f("B"), f("C"),
                            D=x["D"][sl].astype(float), z=f("z")[:, :, sl],
                            delta_bias=x["delta_bias"][sl].astype(float), h0=x["h0"][:, sl].astype(float),
                            nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (lo, hi, o, st))
        q.put((rank, got, mx, rate, parts))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from selective_state_space_36_b200 import inputs as I
    import bench
    assert bench.rank_config(0) == I.MAMBA1P4B
    small = I.ScanConfig("shard", 2, 40, 12, 4, io="bf16", seed=3, h0_sigma=0.2)
    x = I.scan_inputs(small)
    f = lambda k: I.to_f64(x[k], "bf16")
    full_o, full_st = oracle.scan(f("u"), f("delta"), x["A"].astype(float), f("B"), f("C"),
                                  D=x["D"].astype(float), z=f("z"), delta_bias=x["delta_bias"].astype(float),
                                  h0=x["h0"].astype(float), nthreads=1)
    for rank, got, mx, rate, parts in res:
        assert got[0] != got[1], "ranks must draw independent inputs"
        assert mx == [11.0, 5.0]
        assert rate == pytest.approx(2 * 1000 / 11e-3 / 1e9)
        o = np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])], axis=2)
        st = np.concatenate([p[3] for p in sorted(parts, key=lambda p: p[0])], axis=1)
        assert np.array_equal(o, full_o) and np.array_equal(st, full_st)
