"""The benchmark's multi-rank path on CPU: two gloo ranks run the whole-job
aggregation (max of per-rank times, sum of per-rank work) that a multi-GPU run
does over NCCL; the data path itself has no collective (independent batches)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ms_local = [10.0, 12.5][rank]
    bytes_local = [1000, 3000][rank]
    ms, gbs, tps = bench.aggregate(ms_local, bytes_local, 7, steps=4, world=world, device="cpu")
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, ms, gbs, tps))


def test_two_rank_aggregation_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for _, ms, gbs, tps in res:
        assert ms == 12.5                                    # slowest rank
        assert gbs == pytest.approx((1000 + 3000) * 4 / 12.5e-3 / 1e9)
        assert tps == pytest.approx(2 * 7 * 4 / 12.5e-3)


def test_step_bytes_formula():
    import bench
    b = bench.step_bytes(R=8, T=4096, H=7168, K=8, N=171362)
    X, Y = 8 * 4096 * 7168 * 2, 171362 * 7168 * 2
    assert b["dispatch"] >= X + Y and b["combine"] >= X + Y
    assert b["step"] == b["layout"] + b["scan"] + b["dispatch"] + b["combine"]
