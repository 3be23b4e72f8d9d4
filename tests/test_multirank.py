"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on CPU:
every rank draws its own request batch (no data-path collective), the step
time is the max over ranks, and the throughput counts every rank's requests."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        t = bench.reduce_max(1.5 + rank, "cpu")     # this rank's step time (ms)
        bench.barrier()
        seed = bench.rank_seed(0, r)
        q.put((r, ws, t, seed, bench.weak_value(ws, 8, t)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_time_and_draw_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [x[1] for x in res] == [2, 2]
    assert [x[2] for x in res] == [2.5, 2.5]             # max over ranks
    assert res[0][3] != res[1][3]                       # independent request batches
    assert res[0][4] == res[1][4] == pytest.approx(2 * 8 / 2.5e-3)


def test_single_process_defaults():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_env() == (1, 0, 0)
    assert bench.reduce_max(3.0, "cpu") == 3.0
