"""Sharded exchange: the R virtual ranks spread over W GPUs (one shard per GPU).

Argument marshalling and the host-side protocol only; the layout, handle scan,
dispatch (rows written straight into the receive buffers of the GPU hosting
each destination) and combine (rows read back from there) run in libep.so's
kernels (``ep_create_sharded``, ``ep_sharded_handle``, ``ep_sharded_dispatch``,
``ep_sharded_combine``; see include/ep.h).

Shard w hosts virtual ranks [w*R/W, (w+1)*R/W): their tokens, their experts
and the receive buffers of those ranks.  DeepEP's ranks are GPUs joined by
NVLink whose buffers are allocated per rank and shared by exchanging IPC
handles ("DeepEP Buffer Class API ...", section "Construction and Resource
Allocation"); here each shard's receive buffers are registered allocations
(``ep_shared_alloc``) that the other shards map (``ep_ipc_open``).

Two ways to run the W shards:
  * ``ProcessShardGroup``: one process per GPU, ``torch.distributed`` for the
    count all-gather, the handle exchange and the two barriers of a step;
  * ``LocalShardGroup``: all W shards in one process on one device, their
    pointer tables wired directly.  Every shard's kernels run one after the
    other on one stream, and none waits on another, so this exercises the
    sharded kernels' addressing exactly, without several GPUs.
"""
from __future__ import annotations

import ctypes

import torch

from . import (_check, _event, _i64, _ptr, _stream, _vp, ep_config, ep_destroy, ep_get_dispatch_layout,
               load)

IPC_HANDLE_BYTES = 64


def shard_ranks(num_ranks: int, num_shards: int, shard: int) -> tuple[int, int]:
    """(first rank, rank count) hosted by `shard`."""
    if num_shards < 1 or num_ranks % num_shards != 0 or not 0 <= shard < num_shards:
        raise ValueError(f"{num_ranks} ranks cannot be split into {num_shards} equal shards "
                         f"(shard {shard})")
    per = num_ranks // num_shards
    return shard * per, per


def pointer_table(own: int, peers: dict[int, int], shard: int, num_shards: int) -> list[int]:
    """Device pointers of one buffer for every shard, in shard order: this
    process's own buffer at its own index, the mapped peers' elsewhere."""
    table = []
    for w in range(num_shards):
        p = own if w == shard else peers.get(w)
        if not p:
            raise ValueError(f"no pointer for shard {w}")
        table.append(p)
    return table


def _table(ptrs):
    if ptrs is None:
        return None
    arr = (_vp * len(ptrs))(*[_vp(p) for p in ptrs])
    return ctypes.cast(arr, ctypes.POINTER(_vp)), arr   # keep arr alive with the pointer


class _DeviceView:
    """A raw device allocation seen by torch (``__cuda_array_interface__``, no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


_TYPESTR = {torch.bfloat16: "<i2", torch.int64: "<i8", torch.float32: "<f4", torch.int32: "<i4"}


def _view(ptr: int, shape, dtype, device) -> torch.Tensor:
    t = torch.as_tensor(_DeviceView(ptr, shape, _TYPESTR[dtype]), device=device)
    return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t


def shared_alloc(shape, dtype, device):
    """A registered device buffer: (tensor, device pointer, IPC handle bytes)."""
    n = 1
    for d in shape:
        n *= d
    nbytes = max(n, 1) * torch.empty((), dtype=dtype).element_size()
    ptr = _vp()
    handle = (ctypes.c_uint8 * IPC_HANDLE_BYTES)()
    with torch.cuda.device(device):
        _check(load().ep_shared_alloc(nbytes, ctypes.byref(ptr), handle), "ep_shared_alloc")
    return _view(ptr.value, shape, dtype, device), ptr.value, bytes(handle)


def ipc_open(handle: bytes, device) -> int:
    buf = (ctypes.c_uint8 * IPC_HANDLE_BYTES).from_buffer_copy(handle)
    ptr = _vp()
    with torch.cuda.device(device):
        _check(load().ep_ipc_open(buf, ctypes.byref(ptr)), "ep_ipc_open")
    return ptr.value


class ShardedBuffer:
    """One shard of a sharded exchange: its context, its registered receive
    buffers (rows, top-k ids, weights, source indices, expert outputs y) and its
    per-step arrays.  ``connect`` gives it every shard's buffer pointers."""

    BUFFERS = ("recv_x", "recv_idx", "recv_w", "recv_src", "y")

    def __init__(self, num_ranks, num_experts, num_tokens, hidden, topk, num_shards, shard,
                 capacity, num_channels=10, device=None):
        self.device = (torch.device("cuda", torch.cuda.current_device()) if device is None
                       else torch.device(device))
        self.R, self.E, self.T, self.H, self.K = num_ranks, num_experts, num_tokens, hidden, topk
        self.W, self.shard = num_shards, shard
        self.r0, self.Rl = shard_ranks(num_ranks, num_shards, shard)
        self.L = num_experts // num_ranks
        self.capacity = capacity
        cfg = ep_config(num_ranks, num_experts, num_tokens, hidden, topk, num_channels, 0)
        ctx = _vp()
        with torch.cuda.device(self.device):
            _check(load().ep_create_sharded(ctypes.byref(cfg), num_shards, shard, ctypes.byref(ctx)),
                   "ep_create_sharded")
        self.ctx = ctx
        cap = max(capacity, 1)
        shapes = {"recv_x": ((cap, hidden), torch.bfloat16), "recv_idx": ((cap, topk), torch.int64),
                  "recv_w": ((cap, topk), torch.float32), "recv_src": ((cap,), torch.int32),
                  "y": ((cap, hidden), torch.bfloat16)}
        self._own_ptr, self.handles, self._opened = {}, {}, []
        for name, (shape, dtype) in shapes.items():
            t, ptr, h = shared_alloc(shape, dtype, self.device)
            setattr(self, name, t)
            self._own_ptr[name] = ptr
            self.handles[name] = h
        self.tables = None
        dev = dict(device=self.device)
        Rl, T, R, E = self.Rl, num_tokens, num_ranks, num_experts
        self.tin = torch.empty((Rl, T, R), dtype=torch.uint8, **dev)
        self.ntr = torch.empty((Rl, R), dtype=torch.int32, **dev)
        self.nte = torch.empty((Rl, E), dtype=torch.int32, **dev)
        self.ntr_all = torch.empty((R, R), dtype=torch.int32, **dev)
        self.nte_all = torch.empty((R, E), dtype=torch.int32, **dev)
        self.send_head = torch.empty((Rl, T, R), dtype=torch.int32, **dev)
        self.dst_offset = torch.empty((R,), dtype=torch.int64, **dev)
        self.num_recv_rows = torch.empty((1,), dtype=torch.int64, **dev)
        self.num_recv_tokens_per_expert = torch.empty((Rl, self.L), dtype=torch.int32, **dev)

    # -------------------------------------------------------------- wiring
    def connect(self, peer_ptrs: dict[int, dict[str, int]]):
        """peer_ptrs[w][name]: device pointer (valid here) of shard w's buffer."""
        self.tables = {name: pointer_table(self._own_ptr[name], {w: p[name] for w, p in peer_ptrs.items()},
                                           self.shard, self.W)
                       for name in self.BUFFERS}

    def open_peers(self, all_handles: list[dict[str, bytes]]):
        """Map the other shards' registered buffers from their IPC handles."""
        peers = {}
        for w, hs in enumerate(all_handles):
            if w == self.shard:
                continue
            peers[w] = {}
            for name in self.BUFFERS:
                ptr = ipc_open(hs[name], self.device)
                self._opened.append(ptr)
                peers[w][name] = ptr
        self.connect(peers)

    def own_pointers(self) -> dict[str, int]:
        return dict(self._own_ptr)

    # -------------------------------------------------------------- step
    def layout(self, topk_idx, stream=None):
        ep_get_dispatch_layout(self.ctx, topk_idx, self.ntr, self.nte, self.tin, stream)

    def handle(self, stream=None, wait_event=None):
        """send_head, dst_offset, num_recv_rows, per-expert counts from the gathered counts."""
        _check(load().ep_sharded_handle(self.ctx, _ptr(self.tin), _ptr(self.ntr_all), _ptr(self.nte_all),
                                        _ptr(self.send_head), _ptr(self.dst_offset), _ptr(self.num_recv_rows),
                                        _ptr(self.num_recv_tokens_per_expert), _stream(stream),
                                        _event(wait_event)), "ep_sharded_handle", self.ctx)

    def dispatch_rows(self, x, topk_idx, topk_weights=None, stream=None, wait_event=None):
        if self.tables is None:
            raise RuntimeError("connect the shards first")
        tx, ax = _table(self.tables["recv_x"])
        ti, ai = _table(self.tables["recv_idx"])
        tw, aw = _table(self.tables["recv_w"]) if topk_weights is not None else (None, None)
        ts, as_ = _table(self.tables["recv_src"])
        _check(load().ep_sharded_dispatch(self.ctx, _ptr(x), _ptr(topk_idx), _ptr(topk_weights),
                                          _ptr(self.send_head), _ptr(self.dst_offset), self.W, tx, ti, tw, ts,
                                          self.capacity, _stream(stream), _event(wait_event)),
               "ep_sharded_dispatch", self.ctx)

    def combine(self, out_x, out_topk_weights=None, bias=(None, None), stream=None, wait_event=None):
        if self.tables is None:
            raise RuntimeError("connect the shards first")
        ty, ay = _table(self.tables["y"])
        tw, aw = _table(self.tables["recv_w"]) if out_topk_weights is not None else (None, None)
        _check(load().ep_sharded_combine(self.ctx, self.W, ty, tw, self.capacity, _ptr(self.send_head),
                                         _ptr(self.dst_offset), _ptr(bias[0]), _ptr(bias[1]), _ptr(out_x),
                                         _ptr(out_topk_weights), _stream(stream), _event(wait_event)),
               "ep_sharded_combine", self.ctx)

    def received(self):
        """This shard's receive rows: (num rows, recv_x, recv_idx, recv_w, recv_src) views."""
        n = int(self.num_recv_rows.item())
        return n, self.recv_x[:n], self.recv_idx[:n], self.recv_w[:n], self.recv_src[:n]

    def sync_status(self) -> int:
        return load().ep_sync_status(self.ctx, _stream())

    def destroy(self):
        lib = load()
        for p in self._opened:
            lib.ep_ipc_close(_vp(p))
        self._opened = []
        for p in self._own_ptr.values():
            lib.ep_shared_free(_vp(p))
        self._own_ptr = {}
        if self.ctx is not None:
            ep_destroy(self.ctx)
            self.ctx = None


class LocalShardGroup:
    """W shards in one process on one device, run one after the other.  The
    step is the multi-GPU one with the barriers replaced by stream order."""

    def __init__(self, num_ranks, num_experts, num_tokens, hidden, topk, num_shards, capacity,
                 num_channels=10, device=None):
        self.shards = [ShardedBuffer(num_ranks, num_experts, num_tokens, hidden, topk, num_shards, w, capacity,
                                     num_channels, device) for w in range(num_shards)]
        ptrs = {w: b.own_pointers() for w, b in enumerate(self.shards)}
        for w, b in enumerate(self.shards):
            b.connect({v: p for v, p in ptrs.items() if v != w})

    def dispatch(self, xs, topks, weights=None):
        """xs[w] [Rl][T][H], topks[w] [Rl][T][K], weights[w] (or None) per shard."""
        for b, t in zip(self.shards, topks):
            b.layout(t)
        ntr_all = torch.cat([b.ntr for b in self.shards])
        nte_all = torch.cat([b.nte for b in self.shards])
        for b in self.shards:
            b.ntr_all.copy_(ntr_all)
            b.nte_all.copy_(nte_all)
            b.handle()
        for w, b in enumerate(self.shards):
            b.dispatch_rows(xs[w], topks[w], None if weights is None else weights[w])

    def combine(self, outs, out_ws=None, biases=None):
        for w, b in enumerate(self.shards):
            b.combine(outs[w], None if out_ws is None else out_ws[w],
                      (None, None) if biases is None else biases[w])

    def destroy(self):
        for b in self.shards:
            b.destroy()


def exchange_handles(group, handles: dict[str, bytes], num_shards: int) -> list[dict[str, bytes]]:
    """Every shard's registered-buffer IPC handles, in shard (= group rank) order."""
    import torch.distributed as dist
    out = [None] * num_shards
    dist.all_gather_object(out, handles, group=group)
    return out


def gather_counts(group, ntr: torch.Tensor, nte: torch.Tensor, ntr_all: torch.Tensor, nte_all: torch.Tensor):
    """All shards' layout counts ([Rl][R] and [Rl][E] each), in shard order, into
    ntr_all [R][R] / nte_all [R][E].  NCCL gathers device tensors directly; other
    backends go through host memory."""
    import torch.distributed as dist
    if ntr.is_cuda and dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(ntr_all, ntr, group=group)
        dist.all_gather_into_tensor(nte_all, nte, group=group)
        return
    world = dist.get_world_size(group)
    for local, full in ((ntr, ntr_all), (nte, nte_all)):
        parts = [torch.empty_like(local, device="cpu") for _ in range(world)]
        dist.all_gather(parts, local.cpu(), group=group)
        full.copy_(torch.cat(parts))


class ProcessShardGroup:
    """This process's shard of a W-process exchange over `group` (one GPU each).
    Collective steps are taken in the same order on every rank."""

    def __init__(self, group, buffer: ShardedBuffer):
        import torch.distributed as dist
        self.dist, self.group, self.buf = dist, group, buffer
        if dist.get_world_size(group) != buffer.W or dist.get_rank(group) != buffer.shard:
            raise ValueError("one process per shard: group rank w hosts shard w")
        buffer.open_peers(exchange_handles(group, buffer.handles, buffer.W))

    def barrier(self):
        torch.cuda.current_stream(self.buf.device).synchronize()
        self.dist.barrier(group=self.group)

    def gather_counts(self):
        gather_counts(self.group, self.buf.ntr, self.buf.nte, self.buf.ntr_all, self.buf.nte_all)

    def dispatch(self, x, topk_idx, topk_weights=None):
        """Layout, count exchange, handle, rows into every shard; returns after
        every shard's rows have landed (barrier)."""
        b = self.buf
        b.layout(topk_idx)
        self.gather_counts()
        b.handle()
        b.dispatch_rows(x, topk_idx, topk_weights)
        self.barrier()

    def combine(self, out_x, out_topk_weights=None, bias=(None, None)):
        """Call after this shard's expert outputs are in `buf.y`: waits until
        every shard's are, then reduces."""
        self.barrier()
        self.buf.combine(out_x, out_topk_weights, bias)
