"""The multi-process path of bench.py on CPU: two and three gloo ranks.

bench.py runs one global workload whose batch rows are split over the ranks
by selective_state_space_36_b200.shard.scan_shard (channels of every row when
there are fewer rows than ranks); rows are drawn by their global index, and
there is no exchange on the data path.  Here each rank takes its shard of
small problems with the same partition code, scans it with the fp64 oracle,
and the gathered outputs and states must equal one process scanning the whole
problem bit for bit.  The timing reduction (maximum over ranks) and the
whole-job rate are checked too.
"""
import os
import socket
from types import SimpleNamespace

import numpy as np
import pytest
import torch.multiprocessing as mp

from selective_state_space_36_b200.shard import Shard, scan_shard

SMALL = [dict(name="rows", batch=4, seqlen=40, dim=24, dstate=4),      # batch >= ranks: rows split
         dict(name="channels", batch=1, seqlen=33, dim=40, dstate=16)]  # batch < ranks: channels split


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _small_cfg(c):
    from selective_state_space_36_b200 import inputs as I
    return I.ScanConfig(c["name"], c["batch"], c["seqlen"], c["dim"], c["dstate"], io="bf16", seed=3, h0_sigma=0.2)


def _oracle_on(cfg, sh: Shard):
    """The oracle on rows [b0, b1), channels [d0, d1) of cfg, drawn by their
    global indices (as bench.py draws a rank's share)."""
    import oracle
    from selective_state_space_36_b200 import inputs as I
    x = I.scan_inputs(cfg)
    f = lambda k: I.to_f64(x[k], "bf16")
    rs, cs = slice(sh.b0, sh.b1), slice(sh.d0, sh.d1)
    return oracle.scan(f("u")[rs, :, cs], f("delta")[rs, :, cs], x["A"][cs].astype(float), f("B")[rs],
                       f("C")[rs], D=x["D"][cs].astype(float), z=f("z")[rs, :, cs],
                       delta_bias=x["delta_bias"][cs].astype(float), h0=x["h0"][rs, cs].astype(float),
                       nthreads=1)


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        args = SimpleNamespace(workload="mamba1p4b", batch=0, seqlen=0)
        gcfg, sh = bench.sharded_workload(args, rank, world)
        parts = {}
        for c in SMALL:
            cfg = _small_cfg(c)
            s = scan_shard(cfg.batch, cfg.dim, world, rank)
            o, st = _oracle_on(cfg, s)
            got = [None] * world
            dist.all_gather_object(got, (s, o, st))
            parts[c["name"]] = got
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank])
        q.put((rank, gcfg, sh, parts, mx))
    finally:
        dist.destroy_process_group()


def test_scan_shard_covers_the_workload_once():
    for batch, dim, world in [(8, 4096, 1), (16, 4096, 2), (8, 4096, 8), (5, 1536, 3), (1, 1536, 8),
                              (3, 100, 4), (2, 7, 3)]:
        seen = np.zeros((batch, dim), dtype=int)
        for r in range(world):
            s = scan_shard(batch, dim, world, r)
            seen[s.b0:s.b1, s.d0:s.d1] += 1
            if batch < world and s.d1 < dim:
                assert s.d1 % 8 == 0  # channel blocks keep 16-byte aligned bf16 rows
        assert np.all(seen == 1), (batch, dim, world)


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_the_one_process_result(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from selective_state_space_36_b200 import inputs as I
    full = {c["name"]: _oracle_on(_small_cfg(c), Shard(0, c["batch"], 0, c["dim"])) for c in SMALL}
    rows_seen = set()
    for rank, gcfg, sh, parts, mx in res:
        # the benchmark's global workload: the 1.4B-layer shape with world x 8 rows
        assert gcfg.batch == I.MAMBA1P4B.batch * world and gcfg.dim == I.MAMBA1P4B.dim
        assert (sh.d0, sh.d1) == (0, gcfg.dim)
        rows_seen |= set(range(sh.b0, sh.b1))
        assert mx == [10.0 + world - 1, 5.0]
        for c in SMALL:
            fo, fs = full[c["name"]]
            o, st = np.zeros_like(fo), np.zeros_like(fs)
            for s, po, pst in parts[c["name"]]:
                o[s.b0:s.b1, :, s.d0:s.d1] = po
                st[s.b0:s.b1, s.d0:s.d1] = pst
            assert np.array_equal(o, fo) and np.array_equal(st, fs), c["name"]
    assert rows_seen == set(range(I.MAMBA1P4B.batch * world))
