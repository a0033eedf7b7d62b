"""Host logic of `bench.py --gpus N` (independent replicas, no data-path
collective): rank setup from the torchrun environment, the barrier around the
timed region and the max-over-ranks time, exercised with two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import bench
    w, r, local, pg = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank) and pg is not None
    bench.barrier(pg, "cpu")
    t = bench.reduce_max(pg, 1.0 + 2.5 * rank, "cpu")   # per-rank step time in ms
    bench.barrier(pg, "cpu")
    out[rank] = t
    pg.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, _free_port() if r < 0 else port, out))
                 for port in [_free_port()] for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert dict(out) == {0: 3.5, 1: 3.5}
