"""Sharded exchange (the virtual ranks spread over W GPUs) against the one-GPU
oracle: the whole problem's send_head, receive rows, metadata and combine must
come out bit-identical, only placed in the receive buffer of the shard hosting
each destination.  On one device: (a) W shards in one process (LocalShardGroup:
the kernels run one after the other and none waits on another), (b) two
processes exchanging CUDA IPC handles over gloo (ProcessShardGroup), with host
barriers between the steps."""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from helpers import Inputs, bf16_abs, check_combine, to_bf16_tensor, u16

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = [
    (W["dsv3"].scaled(num_tokens=300, hidden=512), 2),
    (W["dsv3"].scaled(num_tokens=300, hidden=512), 4),
    (W["dsv3"].scaled(num_tokens=300, hidden=512), 8),     # one virtual rank per GPU
    (W["zipf"].scaled(num_tokens=60, hidden=256), 4),      # 32 ranks, skewed destinations
    (synth.Workload("odd", 4, 12, 70, 40, 3, "uniform_masked", 83, num_channels=3, mask_prob=0.3), 2),
    (synth.Workload("one-shard", 4, 8, 50, 64, 2, "uniform", 82, num_channels=2), 1),
]


def ids(cases):
    return [f"{w.name}-W{n}" for w, n in cases]


@pytest.fixture(scope="module")
def ep(cuda_lib):
    return cuda_lib


def oracle_all(inp):
    w = inp.w
    ntr, nte, tin = oracle.layout(inp.topk, w.num_experts)
    h = oracle.dispatch_handle(tin, nte, w.num_channels)
    rows = oracle.dispatch_rows(inp.x_u16, inp.topk, inp.weights, h, w.num_experts)
    return tin, h, rows


def shard_offsets(h, R, nshards):
    """From the oracle's receive offsets: rows per destination, each destination's
    first row inside its shard's buffer, rows per shard."""
    off = h["recv_rank_offset"]
    n = np.diff(off)
    per = R // nshards
    dst = np.zeros(R, dtype=np.int64)
    for d in range(R):
        first = d // per * per
        dst[d] = n[first:d].sum()
    rows = [int(n[s * per:(s + 1) * per].sum()) for s in range(nshards)]
    return n, dst, rows


def check_dispatch(ep, w, nshards, shards, inp, tin, h, rows):
    o_x, o_idx, o_w = rows
    R, per = w.num_ranks, w.num_ranks // nshards
    n, dst, shard_rows = shard_offsets(h, R, nshards)
    off = h["recv_rank_offset"]
    for s, b in enumerate(shards):
        r0 = s * per
        np.testing.assert_array_equal(b.tin.cpu().numpy(), tin[r0:r0 + per], err_msg="is_token_in_rank")
        np.testing.assert_array_equal(b.send_head.cpu().numpy(), h["send_head"][r0:r0 + per], err_msg="send_head")
        np.testing.assert_array_equal(b.dst_offset.cpu().numpy(), dst, err_msg="dst_offset")
        assert int(b.num_recv_rows.item()) == shard_rows[s]
        np.testing.assert_array_equal(b.num_recv_tokens_per_expert.cpu().numpy(),
                                      h["num_recv_tokens_per_expert"][r0:r0 + per])
        rx, ri, rw, rs = (u16(b.recv_x), b.recv_idx.cpu().numpy(), b.recv_w.cpu().numpy(),
                          b.recv_src.cpu().numpy())
        for d in range(r0, r0 + per):
            a, z = int(dst[d]), int(dst[d] + n[d])
            np.testing.assert_array_equal(rx[a:z], o_x[off[d]:off[d + 1]], err_msg=f"rows of rank {d}")
            np.testing.assert_array_equal(ri[a:z], o_idx[off[d]:off[d + 1]], err_msg=f"ids of rank {d}")
            np.testing.assert_array_equal(rw[a:z], o_w[off[d]:off[d + 1]], err_msg=f"weights of rank {d}")
            np.testing.assert_array_equal(rs[a:z], h["recv_src_idx"][off[d]:off[d + 1]], err_msg=f"src of {d}")
    return n, dst


@pytest.mark.parametrize("case", CASES, ids=ids(CASES))
def test_local_shards_match_one_gpu(ep, case):
    from combine_ep_get_11_b200 import sharded
    w, nshards = case
    inp = Inputs(w)
    tin, h, rows = oracle_all(inp)
    R, T, H, K = w.num_ranks, w.num_tokens, w.hidden, w.topk
    per = R // nshards
    n, dst, shard_rows = shard_offsets(h, R, nshards)
    cap = max(shard_rows) + 5
    group = sharded.LocalShardGroup(R, w.num_experts, T, H, K, nshards, cap, w.num_channels)
    sl = [slice(s * per, (s + 1) * per) for s in range(nshards)]
    group.dispatch([inp.x_d[q] for q in sl], [inp.topk_d[q] for q in sl], [inp.weights_d[q] for q in sl])
    for b in group.shards:
        assert b.sync_status() == 0
    check_dispatch(ep, w, nshards, group.shards, inp, tin, h, rows)

    # identity experts: the combine is exact, so bit-identical to the oracle's
    for b in group.shards:
        b.y.copy_(b.recv_x)
    outs = [torch.empty((per, T, H), dtype=torch.bfloat16, device="cuda") for _ in range(nshards)]
    out_ws = [torch.empty((per, T, K), dtype=torch.float32, device="cuda") for _ in range(nshards)]
    group.combine(outs, out_ws)
    e_out, e_w = oracle.combine(rows[0], h, rows[2])
    for s in range(nshards):
        np.testing.assert_array_equal(u16(outs[s]), e_out[sl[s]])
        np.testing.assert_array_equal(out_ws[s].cpu().numpy(), e_w[sl[s]])

    # independent expert outputs (placed row for row as received) and two bias terms:
    # N(0,1) rows, then rows whose large terms cancel (the rank order shows)
    N = int(h["recv_rank_offset"][-1])
    off = h["recv_rank_offset"]
    b0, b1 = synth.bias_rows(w, 0), synth.bias_rows(w, 1)
    bias = dict(bias0=u16(b0), bias1=u16(b1))
    for what, y in (("N(0,1) rows", u16(synth.expert_rows(w.seed + 5, N, H))),
                    ("cancelling rows", synth.cancel_rows(w.seed + 6, N, H))):
        for s, b in enumerate(group.shards):
            for d in range(s * per, (s + 1) * per):
                b.y[int(dst[d]):int(dst[d] + n[d])].copy_(to_bf16_tensor(y[off[d]:off[d + 1]]).cuda())
        group.combine(outs, None, [(b0[q].cuda(), b1[q].cuda()) for q in sl])
        got = np.concatenate([u16(o) for o in outs])
        check_combine(f"{w.name} over {nshards} shards: combine, {what} + 2 biases", got,
                      oracle.combine(y, h, fp32=True, **bias)[0], oracle.combine(y, h, **bias)[0],
                      oracle.combine(bf16_abs(y), h, bias0=bf16_abs(bias["bias0"]),
                                     bias1=bf16_abs(bias["bias1"]))[0], min(R, K) + 2,
                      one_ulp=what == "N(0,1) rows", cancelling=what == "cancelling rows")
    for b in group.shards:
        assert b.sync_status() == 0
    group.destroy()


def test_sharded_refusals_and_capacity(ep):
    from combine_ep_get_11_b200 import EpError, sharded
    w = W["dsv3"].scaled(num_tokens=64, hidden=64)
    with pytest.raises(ValueError):     # 8 ranks do not split into 3 shards
        sharded.ShardedBuffer(w.num_ranks, w.num_experts, w.num_tokens, w.hidden, w.topk, 3, 0, 16)
    inp = Inputs(w)
    group = sharded.LocalShardGroup(w.num_ranks, w.num_experts, w.num_tokens, w.hidden, w.topk, 2, 8)
    b = group.shards[0]
    # the single-GPU calls are refused on a sharded context
    handle = ep.Handle.empty(w.num_ranks, w.num_tokens, w.num_channels, w.local_experts, 8, "cuda")
    with pytest.raises(EpError):
        ep.ep_dispatch(b.ctx, inp.x_d[:4], inp.topk_d[:4], None, None, None, None, handle,
                       torch.empty((8, w.hidden), dtype=torch.bfloat16, device="cuda"), None, None, 8)
    with pytest.raises(EpError):          # a shard's receive count comes from ep_sharded_handle
        ep.ep_get_num_recv(b.ctx, torch.zeros((4, 8), dtype=torch.int32, device="cuda"), 8)
    # receive buffers of 8 rows are far too small: rows past them are dropped and reported
    group.dispatch([inp.x_d[:4], inp.x_d[4:]], [inp.topk_d[:4], inp.topk_d[4:]])
    assert b.sync_status() == 3          # EP_ERR_CAPACITY
    assert group.shards[1].sync_status() == 3
    group.destroy()


# ------------------------------------------------------------ two processes, CUDA IPC

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


IPC_CASE = W["dsv3"].scaled(num_tokens=200, hidden=256)


def _ipc_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    from combine_ep_get_11_b200 import EpError, sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    w = IPC_CASE
    inp = Inputs(w)
    R, per = w.num_ranks, w.num_ranks // world
    sl = slice(rank * per, (rank + 1) * per)
    # every token of every rank could go to each of the shard's ranks
    buf = sharded.ShardedBuffer(R, w.num_experts, w.num_tokens, w.hidden, w.topk, world, rank,
                                capacity=w.num_tokens * R * per, num_channels=w.num_channels)
    try:
        grp = sharded.ProcessShardGroup(dist.group.WORLD, buf)
        ok = torch.tensor([1])
    except EpError as e:      # CUDA IPC not available here
        ok = torch.tensor([0])
        msg = str(e)
    dist.all_reduce(ok, op=dist.ReduceOp.MIN)
    if not ok.item():
        buf.destroy()
        dist.destroy_process_group()
        q.put((rank, "unavailable", msg if "msg" in locals() else "a peer could not map the buffers"))
        return
    grp.dispatch(inp.x_d[sl].contiguous(), inp.topk_d[sl].contiguous(), inp.weights_d[sl].contiguous())
    n = int(buf.num_recv_rows.item())
    buf.y[:n].copy_(buf.recv_x[:n])                     # identity experts
    out = torch.empty((per, w.num_tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    out_w = torch.empty((per, w.num_tokens, w.topk), dtype=torch.float32, device="cuda")
    grp.combine(out, out_w)
    torch.cuda.synchronize()
    status = buf.sync_status()
    res = dict(status=status, send_head=buf.send_head.cpu().numpy(), dst=buf.dst_offset.cpu().numpy(),
               rows=u16(buf.recv_x[:n]), src=buf.recv_src[:n].cpu().numpy(), out=u16(out),
               out_w=out_w.cpu().numpy())
    dist.barrier()                      # no shard unmaps while another still reads
    buf.destroy()
    dist.destroy_process_group()
    q.put((rank, "ok", res))


def test_two_processes_over_cuda_ipc(ep):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = []
    for _ in range(world):
        results.append(q.get(timeout=300))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    results.sort(key=lambda r: r[0])
    if any(r[1] == "unavailable" for r in results):
        pytest.skip(f"CUDA IPC between processes unavailable: {results[0][2]}")
    w = IPC_CASE
    inp = Inputs(w)
    tin, h, rows = oracle_all(inp)
    R, per = w.num_ranks, w.num_ranks // world
    n, dst, _ = shard_offsets(h, R, world)
    off = h["recv_rank_offset"]
    e_out, e_w = oracle.combine(rows[0], h, rows[2])
    for rank, _, res in results:
        assert res["status"] == 0
        sl = slice(rank * per, (rank + 1) * per)
        np.testing.assert_array_equal(res["send_head"], h["send_head"][sl])
        np.testing.assert_array_equal(res["dst"], dst)
        for d in range(rank * per, (rank + 1) * per):
            a, z = int(dst[d]), int(dst[d] + n[d])
            np.testing.assert_array_equal(res["rows"][a:z], rows[0][off[d]:off[d + 1]])
            np.testing.assert_array_equal(res["src"][a:z], h["recv_src_idx"][off[d]:off[d + 1]])
        np.testing.assert_array_equal(res["out"], e_out[sl])
        np.testing.assert_array_equal(res["out_w"], e_w[sl])
