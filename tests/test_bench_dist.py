"""The benchmark's multi-rank host side on CPU: two gloo ranks run the whole-job
aggregation (max of per-rank times, sum of per-rank work) that a multi-GPU run
does over NCCL, for independent replicas and for the sharded exchange (each rank
holding half of one problem), and the NVLink byte count of a sharded step."""
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
    b = bench.step_bytes(R=8, T=4096, H=7168, K=8, N=171362, E=256)
    X, Y = 8 * 4096 * 7168 * 2, 171362 * 7168 * 2
    assert b["dispatch"] >= X + Y and b["combine"] >= X + Y
    assert b["step"] == b["layout"] + b["scan"] + b["dispatch"] + b["combine"]
    # the layout's histograms grow with the expert count
    assert bench.step_bytes(8, 4096, 7168, 8, 171362, E=512)["layout"] - b["layout"] == 8 * 256 * 4


def test_nvlink_traffic_hand_count():
    """Two GPUs, four ranks (two each): rows leave a GPU for the other GPU's ranks
    in the dispatch and come back in the combine."""
    import numpy as np

    import bench
    ntr = np.array([[5, 1, 2, 0],      # source rank 0 (GPU 0): 2 rows to ranks 2, 3
                    [0, 4, 3, 1],      # source rank 1 (GPU 0): 4
                    [7, 0, 6, 2],      # source rank 2 (GPU 1): 7 to ranks 0, 1
                    [1, 1, 0, 9]])     # source rank 3 (GPU 1): 2
    H, K = 16, 2
    meta = K * 12 + 4
    t0 = bench.nvlink_traffic(ntr, 0, 2, H, K)
    t1 = bench.nvlink_traffic(ntr, 1, 2, H, K)
    assert (t0["rows_out"], t0["rows_in"]) == (6, 9)
    assert (t1["rows_out"], t1["rows_in"]) == (9, 6)
    assert t0["send_bytes"] == 6 * (2 * H + meta) + 9 * (2 * H + 4 * K)
    assert t0["recv_bytes"] == 9 * (2 * H + meta) + 6 * (2 * H + 4 * K)
    assert t0["send_bytes"] == t1["recv_bytes"] and t0["recv_bytes"] == t1["send_bytes"]
    # one GPU: nothing crosses
    t = bench.nvlink_traffic(ntr, 0, 1, H, K)
    assert t["rows_out"] == t["rows_in"] == t["send_bytes"] == t["recv_bytes"] == 0


def _sharded_worker(rank, world, port, q):
    """The sharded benchmark's host side on two gloo ranks: each rank owns half of
    one problem's ranks, its bytes are its share, the job time is the slowest rank's
    and the whole-job figures count the one problem once."""
    import datetime

    import numpy as np
    import torch.distributed as dist

    import bench
    from combine_ep_get_11_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    R, T, H, K, E, N = 8, 64, 32, 4, 16, 1000
    r0, Rl = sharded.shard_ranks(R, world, rank)
    full = bench.step_bytes(R, T, H, K, N, E)
    share = {k: v * Rl / R for k, v in full.items() if k != "step"}
    ms = [4.0, 5.0][rank]
    _, gbs, tps = bench.aggregate(ms, sum(share.values()), Rl * T, steps=3, world=world, device="cpu")
    ntr = np.arange(R * R).reshape(R, R)
    link = bench.max_over_ranks(float(bench.nvlink_traffic(ntr, rank, world, H, K)["send_bytes"]), world, "cpu")
    dist.destroy_process_group()
    q.put((rank, r0, Rl, gbs, tps, link, full["step"]))


def test_two_rank_sharded_aggregation_gloo():
    import numpy as np

    import bench
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [(r0, Rl) for _, r0, Rl, *_ in res] == [(0, 4), (4, 4)]
    step_bytes = res[0][6]
    ntr = np.arange(64).reshape(8, 8)
    exp_link = max(bench.nvlink_traffic(ntr, w, 2, 32, 4)["send_bytes"] for w in range(2))
    for _, _, _, gbs, tps, link, _ in res:
        assert gbs == pytest.approx(step_bytes * 3 / 5e-3 / 1e9)     # one problem, slowest rank
        assert tps == pytest.approx(8 * 64 * 3 / 5e-3)
        assert link == exp_link
