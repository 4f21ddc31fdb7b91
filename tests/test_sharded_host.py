"""Host side of the sharded exchange on CPU: rank partition, pointer tables, and
the two collectives of a step (IPC-handle exchange, layout-count all-gather) run
by two gloo ranks, as the GPU processes run them over NCCL or gloo."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from combine_ep_get_11_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_ranks():
    assert sharded.shard_ranks(8, 1, 0) == (0, 8)
    assert sharded.shard_ranks(8, 4, 3) == (6, 2)
    assert sharded.shard_ranks(32, 8, 5) == (20, 4)
    for bad in ((8, 3, 0), (8, 2, 2), (8, 2, -1), (8, 0, 0)):
        with pytest.raises(ValueError):
            sharded.shard_ranks(*bad)


def test_pointer_table():
    assert sharded.pointer_table(50, {0: 10, 1: 11, 3: 13}, 2, 4) == [10, 11, 50, 13]
    assert sharded.pointer_table(7, {}, 0, 1) == [7]
    with pytest.raises(ValueError):
        sharded.pointer_table(50, {0: 10, 3: 13}, 2, 4)     # shard 1 missing


def _counts(rank, Rl, R, E):
    """Layout counts a shard would produce: distinct per shard and position."""
    ntr = torch.arange(Rl * R, dtype=torch.int32).reshape(Rl, R) + 1000 * rank
    nte = torch.arange(Rl * E, dtype=torch.int32).reshape(Rl, E) * 3 + 7 * rank
    return ntr, nte


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    R, E = 8, 32
    r0, Rl = sharded.shard_ranks(R, world, rank)
    handles = {name: bytes([rank * 16 + i]) * sharded.IPC_HANDLE_BYTES
               for i, name in enumerate(sharded.ShardedBuffer.BUFFERS)}
    got = sharded.exchange_handles(dist.group.WORLD, handles, world)
    ntr, nte = _counts(rank, Rl, R, E)
    ntr_all = torch.empty((R, R), dtype=torch.int32)
    nte_all = torch.empty((R, E), dtype=torch.int32)
    sharded.gather_counts(dist.group.WORLD, ntr, nte, ntr_all, nte_all)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, ntr_all.numpy(), nte_all.numpy()))


def test_exchange_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted((q.get(timeout=10) for _ in range(world)), key=lambda r: r[0])
    R, E, Rl = 8, 32, 4
    exp_ntr = np.concatenate([_counts(w, Rl, R, E)[0].numpy() for w in range(world)])
    exp_nte = np.concatenate([_counts(w, Rl, R, E)[1].numpy() for w in range(world)])
    for rank, got, ntr_all, nte_all in res:
        assert len(got) == world
        for w in range(world):                      # handles in shard order
            for i, name in enumerate(sharded.ShardedBuffer.BUFFERS):
                assert got[w][name] == bytes([w * 16 + i]) * sharded.IPC_HANDLE_BYTES
        np.testing.assert_array_equal(ntr_all, exp_ntr)   # counts in shard order
        np.testing.assert_array_equal(nte_all, exp_nte)
