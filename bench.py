"""Benchmark: MoE dispatch + combine on virtual EP ranks of one B200.

One step = the whole hot path over one batch of synthetic DeepSeek-V3-shaped
routing (8 virtual ranks, 256 experts, 4096 tokens per rank, hidden 7168 bf16,
top-8 with ~2% masked slots):
    ep_get_dispatch_layout -> ep_dispatch (prefix scan + row scatter, with
    top-k ids and weights) -> ep_combine (y = received rows, i.e. identity
    experts; fp32 rank-ordered reduction + combined weights).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--sharded | --replicas] [--repeats R] [--workload NAME]

Prints one JSON line.  `value` is algorithmic HBM traffic per second (GB/s,
bytes the method must move / device time, inputs resident in HBM), from the
median of R timed replays of the K steps (the minimum rides along); tokens/s,
per-kernel times, the dominant kernel's roofline fraction, an end-to-end
number through host buffers, clocks, a sampled oracle check of the combine and
a CPU-oracle baseline ride along.

With N > 1 (torchrun) the default is the sharded exchange: the one DSv3
problem's 8 virtual ranks are spread over the N GPUs (ep_sharded_*), rows go
straight into the receive buffers of the GPU hosting their destination and
come back inside the combine; the layout counts are all-gathered over NCCL
and two one-element NCCL all-reduces order every GPU's dispatch before any
combine and every combine before the next dispatch (strong scaling: the total
work is fixed).  `--sharded` runs that path on one GPU too (one shard).
`--replicas` instead runs an independent batch per GPU (weak scaling, no
data-path collective).  The time is the max over ranks.  `--impl reference`
times the CPU oracle on a bounded sample of the same workload (there is no
runnable upstream implementation).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

WORKLOAD = "dsv3"
FALLBACK_HBM_GBS = 6650.0
NVLINK_GBS = 770.0             # measured peer copy per direction per GPU on this machine's B200s
L2_BYTES = 126 * 1024 * 1024
CPU_SAMPLE_TOKENS = 2048       # oracle baseline: first 2048 tokens of every rank
CPU_SECONDS = 10.0            # oracle baseline: about this much single-threaded CPU work
CHECK_TOKENS = 512             # sampled tokens of the combine checked against the oracle
LB_EXPERTS = 32                # load-balance workload: 32 local experts ...
LB_EXPERT_ELEMS = 3 * 7168 * 2048   # ... of DeepSeek-V3 size (gate/up/down), bf16
LB_REPLICAS = 8                # ... and 8 redundant replicas
METRIC = "dispatch+combine algorithmic HBM GB/s (tokens/s alongside)"


# ------------------------------------------------------------------ bytes

def step_bytes(R, T, H, K, N, E):
    """Algorithmic bytes of each kernel of one step (what the method must move)."""
    X = R * T * H * 2
    Y = N * H * 2
    G = R * T
    b = {
        "layout": G * K * 8 + G * R + R * R * 4 + R * E * 4,
        "scan": G * R + G * R * 4,
        "dispatch": X + G * R * 4 + G * K * 12 + Y + N * (K * 12 + 4),
        "combine": Y + G * R * 4 + N * K * 4 + X + G * K * 4,
    }
    b["step"] = sum(b.values())
    return b


def nvlink_traffic(ntr_all: np.ndarray, shard: int, num_shards: int, H: int, K: int) -> dict:
    """Bytes one GPU of a sharded exchange moves over NVLink per step.

    ntr_all [R][R]: tokens of source rank s for destination rank d (the gathered
    layout counts).  GPU `shard` hosts ranks [shard*R/W, (shard+1)*R/W).  In the
    dispatch it writes every row of its sources bound for another GPU's ranks
    (row, ids, weights, source index) and receives the rows other GPUs' sources
    send to its ranks; in the combine it reads the first kind back (with their
    weights) and the other GPUs read the second kind.  Returns rows and bytes
    per direction."""
    R = ntr_all.shape[0]
    per = R // num_shards
    mine = np.zeros(R, bool)
    mine[shard * per:(shard + 1) * per] = True
    rows_out = int(ntr_all[mine][:, ~mine].sum())     # my sources -> other GPUs' ranks
    rows_in = int(ntr_all[~mine][:, mine].sum())      # other GPUs' sources -> my ranks
    meta = K * 8 + K * 4 + 4
    send = rows_out * (H * 2 + meta) + rows_in * (H * 2 + K * 4)     # my dispatch writes; peers' combine reads
    recv = rows_in * (H * 2 + meta) + rows_out * (H * 2 + K * 4)     # peers' dispatch writes; my combine reads
    return {"rows_out": rows_out, "rows_in": rows_in, "send_bytes": send, "recv_bytes": recv}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "combine_ep_get_11_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source
    is unchanged since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    if rec.get("source_hash") != source_hash(*rec.get("sources", [])):
        return None
    return rec.get("dram_bytes_per_launch_full")


def spread(values):
    """median / min / max of a list of floats."""
    return {"median": statistics.median(values), "min": min(values), "max": max(values)}


# ----------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.t_start = time.time()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), sm_max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hw_thermal=parts[6], sw_thermal=parts[7],
                                 sw_power=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["sm_max"] for r in rows),
                "power_w_max": max(r["power"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist.get_rank(), world, local
    return 0, 1, 0


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (timing only; not on the data path)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(ms_local: float, bytes_per_step: float, tokens_per_step: int, steps: int, world: int,
              device=None):
    """Whole-job numbers over all ranks: the job time is the slowest rank's, the work
    the sum of every rank's (its own batch, or its share of one sharded problem).
    Returns (ms, GB/s, tokens/s)."""
    ms = max_over_ranks(ms_local, world, device)
    total_bytes = sum_over_ranks(float(bytes_per_step) * steps, world, device)
    total_tokens = sum_over_ranks(float(tokens_per_step) * steps, world, device)
    return ms, total_bytes / (ms / 1e3) / 1e9, total_tokens / (ms / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- CPU arm

def oracle_sample(w: synth.Workload, tokens: int):
    """Run the CPU oracle over a bounded sample of the workload; returns (seconds, bytes, tokens)."""
    import torch

    import oracle
    ws = w.scaled(num_tokens=tokens)
    topk = synth.topk_idx(ws)
    wts = synth.topk_weights(ws)
    x = synth.hidden_rows(ws).view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    ntr, nte, tin = oracle.layout(topk, ws.num_experts)
    h = oracle.dispatch_handle(tin, nte, ws.num_channels)
    recv_x, _, recv_w = oracle.dispatch_rows(x, topk, wts, h, ws.num_experts)
    oracle.combine(recv_x, h, recv_w, fp32=True)
    dt = time.perf_counter() - t0
    N = int(h["recv_rank_offset"][-1])
    b = step_bytes(ws.num_ranks, tokens, ws.hidden, ws.topk, N, ws.num_experts)["step"]
    return dt, b, ws.num_ranks * tokens


def cpu_baseline(w, sample_tokens):
    """The oracle on a bounded sample, repeated until about CPU_SECONDS of work."""
    R, T = w.num_ranks, w.num_tokens
    dt = b = tok = 0
    passes = 0
    while passes < 16 and (passes == 0 or dt < CPU_SECONDS):
        d_, b_, t_ = oracle_sample(w, min(sample_tokens, T))
        dt, b, tok, passes = dt + d_, b + b_, tok + t_, passes + 1
    return {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "tokens_per_s": round(tok / dt, 1), "seconds": round(dt, 2),
            "sample": f"{passes} passes over the first {min(sample_tokens, T)} of {T} "
                      f"tokens of each of the {R} ranks (full hidden/top-k): "
                      f"layout+handle+dispatch rows+combine, single-threaded C++ oracle, "
                      f"host cores: {os.cpu_count()}"}


def combine_check(ep, path, w, x_u16, topk, dev):
    """Sampled tokens of the timed combine (identity experts) and of a combine of
    independent N(0,1) expert outputs, against the oracle: bit-exact against its
    fixed-order fp32 definition, and the error against the exact sum (max bf16
    ulps, max relative error, mean absolute error).  Runs after the timed region."""
    import torch

    import oracle
    R, E, T, H = w.num_ranks, w.num_experts, w.num_tokens, w.hidden
    G = R * T
    _, nte, tin = oracle.layout(topk, E)
    h = oracle.dispatch_handle(tin, nte, w.num_channels)
    rng = np.random.default_rng(w.seed + 77)
    tokens = np.sort(rng.choice(G, size=min(CHECK_TOKENS, G), replace=False))
    tok_d = torch.from_numpy(tokens).to(dev)

    def u16(t):
        return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def stats(got, y_host):
        ref32, _ = oracle.combine(y_host, h, tokens=tokens, fp32=True)
        exact, _ = oracle.combine(y_host, h, tokens=tokens)
        g = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        r = (exact.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        diff = np.abs(g - r)
        a = np.abs(r)
        e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -126.0)
        ulp = np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)
        rel = np.where(a > 0, diff / np.where(a > 0, a, 1.0), np.where(diff > 0, np.inf, 0.0))
        return {"elements": int(got.size), "mismatches_vs_fp32_oracle": int((got != ref32).sum()),
                "max_ulp_vs_exact": float((diff / ulp).max()), "max_rel_err_vs_exact": float(rel.max()),
                "mean_abs_err_vs_exact": float(diff.mean())}

    out = {"tokens": int(tokens.size)}
    # the timed step's output: identity experts, y = the oracle's received rows
    recv_x, _, _ = oracle.dispatch_rows(x_u16, topk, None, h, E)
    out["timed_identity_experts"] = stats(u16(path.out.view(G, H)[tok_d]), recv_x)
    del recv_x
    # independent expert outputs, combined once more (untimed)
    y_d = synth.expert_rows_device(w.seed + 5, path.N, H, device=dev)
    o = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    ep.ep_combine(path.ctx, y_d, path.N, path.handle, None, None, None, o, None)
    out["normal_expert_outputs"] = stats(u16(o.view(G, H)[tok_d]), u16(y_d))
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = synth.WORKLOADS[WORKLOAD]
    tokens = args.cpu_sample_tokens
    for _ in range(args.warmup):
        oracle_sample(w, min(tokens, 64))
    total_s, total_b, total_tok = 0.0, 0, 0
    for _ in range(args.steps):
        dt, b, tok = oracle_sample(w, tokens)
        total_s += dt
        total_b += b
        total_tok += tok
    gbs = total_b / total_s / 1e9
    sample = (f"first {tokens} of {w.num_tokens} tokens of each of the {w.num_ranks} ranks, full "
              f"hidden/top-k; layout+handle+dispatch rows+combine in the single-threaded C++ oracle")
    line = {
        "impl": "reference", "metric": METRIC,
        "value": round(gbs, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_s / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "tokens_per_s": round(total_tok / total_s, 1),
        "config": config_dict(w, l2_note="CPU"),
        "cpu_baseline": {"value": round(gbs, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, l2_note):
    return {"workload": f"{w.name}: {w.num_ranks} virtual ranks, {w.num_experts} experts, "
                        f"{w.num_tokens} tokens/rank, hidden {w.hidden} bf16, top-{w.topk} "
                        f"({w.routing}, mask p={w.mask_prob})",
            "num_ranks": w.num_ranks, "num_experts": w.num_experts, "tokens_per_rank": w.num_tokens,
            "hidden": w.hidden, "topk": w.topk, "num_channels": w.num_channels,
            "l2": l2_note}


# ---------------------------------------------------------------- GPU arm

class Path:
    """One workload's timed step on one GPU: buffers, the step itself and its
    algorithmic bytes."""

    def __init__(self, ep, w, dev, topk_d, wts_d, x_d, fp8=False):
        import torch
        self.ep, self.w, self.dev = ep, w, dev
        R, E, T, H, K, C = w.num_ranks, w.num_experts, w.num_tokens, w.hidden, w.topk, w.num_channels
        self.buf = ep.Buffer(R, E, T, H, K, C, w.max_tokens_per_rank, device=dev)
        ctx = self.ctx = self.buf.ctx
        X, G = R * T * H * 2, R * T
        self.units = G
        self.out = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
        self.out_w = None
        self.handle = None
        if w.name == "ll":
            self.fp8 = fp8
            L, cap = E // R, R * w.tmax
            self.packed = torch.empty((R, L, cap, H), dtype=torch.bfloat16, device=dev)
            self.count = torch.empty((R, L), dtype=torch.int32, device=dev)
            self.src_info = torch.empty((R, L, cap), dtype=torch.int32, device=dev)
            self.layout_range = torch.empty((R, L, R, 2), dtype=torch.int32, device=dev)
            # valid (token, expert) pairs, a token counted once per expert (host-side count)
            t = np.sort(topk_d.cpu().numpy().reshape(-1, K), axis=1)
            S = int(((t >= 0) & np.concatenate([np.ones((t.shape[0], 1), bool),
                                                t[:, 1:] != t[:, :-1]], axis=1)).sum())
            self.N = S
            copy_key = "ll_copy_fp8" if fp8 else "ll_copy"
            row_bytes = H + (H // 128) * 4 if fp8 else H * 2
            self.bytes = {"ll_count": G * K * 12 + S * 4 + E * R * 8,
                          copy_key: X + G * K * 12 + S * row_bytes,
                          "ll_combine": S * H * 2 + S * 4 + X + G * K * 12}
            self.dominant = (copy_key, "ll_combine")
            self.inputs = ("x", "topk", "weights")
            if fp8:
                self.codes = torch.empty((R, L, cap, H), dtype=torch.uint8, device=dev)
                self.scales = torch.empty((R, L, cap, H // 128), dtype=torch.float32, device=dev)

            def step(xd, td, wd, out=None, out_w=None):
                if fp8:
                    # experts would read the FP8 rows; their bf16 outputs sit in `packed`
                    ep.ep_ll_dispatch_fp8(ctx, xd, td, self.codes, self.scales, self.count,
                                          self.src_info, self.layout_range)
                else:
                    ep.ep_ll_dispatch(ctx, xd, td, self.packed, self.count, self.src_info,
                                      self.layout_range)
                ep.ep_ll_combine(ctx, self.packed, td, wd, self.src_info, self.layout_range,
                                 self.out if out is None else out)
            self.step = step
            return
        if w.name == "lb":
            # redundant-expert load balance: weight prefetch + gradient reduction of
            # DeepSeek-V3-sized experts (3 x 7168 x 2048 bf16 per expert)
            E_l, W = LB_EXPERTS, LB_EXPERT_ELEMS
            self.mapping = torch.from_numpy(synth.redundancy_mapping(E_l, LB_REPLICAS, seed=w.seed)).to(dev)
            m = self.mapping.cpu().numpy()
            self.ew = synth.expert_rows_device(w.seed + 1, E_l, W, dev)
            self.red = torch.empty((LB_REPLICAS, W), dtype=torch.bfloat16, device=dev)
            self.grads = synth.expert_rows_device(w.seed + 2, E_l, W, dev)
            self.rgrads = synth.expert_rows_device(w.seed + 3, LB_REPLICAS, W, dev)
            nv = int((m >= 0).sum())
            touched = len(set(m[m >= 0].tolist()))
            self.N = nv
            self.bytes = {"lb_prefetch": 2 * nv * W * 2, "lb_reduce": (2 * touched + nv) * W * 2}
            self.dominant = ("lb_prefetch", "lb_reduce")
            self.inputs = ("x",)
            self.units = E_l          # experts

            def step(xd, td, wd, out=None, out_w=None):
                ep.ep_lb_prefetch_weights(ctx, self.ew, self.mapping, self.red)
                ep.ep_lb_reduce_grads(ctx, self.rgrads, self.mapping, self.grads)
            self.step = step
            return
        ntr = torch.empty((R, R), dtype=torch.int32, device=dev)
        nte = torch.empty((R, E), dtype=torch.int32, device=dev)
        tin = torch.empty((R, T, R), dtype=torch.uint8, device=dev)
        ep.ep_get_dispatch_layout(ctx, topk_d, ntr, nte, tin)
        N = self.N = ep.ep_get_num_recv(ctx, ntr, R)[0]   # receive rows of this routing (sizing read, untimed)
        handle = self.handle = ep.Handle.empty(R, T, C, E // R, N, dev)
        handle.is_token_in_rank = tin
        recv_x = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
        Y = N * H * 2
        if w.name == "reuse":
            # handle built once (untimed); each step reuses it: cached dispatch + combine
            ep.ep_dispatch(ctx, x_d, topk_d, wts_d, ntr, nte, tin, handle, recv_x, None, None, N)
            self.bytes = {"dispatch_cached": X + G * R * 4 + Y, "combine": Y + G * R * 4 + X}
            self.dominant = ("dispatch_cached", "combine")
            self.inputs = ("x",)

            def step(xd, td, wd, out=None, out_w=None):
                ep.ep_dispatch_cached(ctx, xd, handle, recv_x, N)
                ep.ep_combine(ctx, recv_x, N, handle, None, None, None, self.out if out is None else out, None)
            self.step = step
            return
        recv_idx = torch.empty((N, K), dtype=torch.int64, device=dev)
        recv_w = torch.empty((N, K), dtype=torch.float32, device=dev)
        self.out_w = torch.empty((R, T, K), dtype=torch.float32, device=dev)
        self.bytes = step_bytes(R, T, H, K, N, E)
        del self.bytes["step"]
        self.dominant = ("dispatch", "combine")
        self.inputs = ("x", "topk", "weights")

        def step(xd, td, wd, out=None, out_w=None):
            ep.ep_get_dispatch_layout(ctx, td, ntr, nte, tin)
            ep.ep_dispatch(ctx, xd, td, wd, ntr, nte, tin, handle, recv_x, recv_idx, recv_w, N)
            ep.ep_combine(ctx, recv_x, N, handle, recv_w, None, None, self.out if out is None else out,
                          self.out_w if out_w is None else out_w)
        self.step = step

    def sync_status(self):
        return self.buf.sync_status()

    def destroy(self):
        self.buf.destroy()


class ShardedPath:
    """The problem's step through the sharded exchange, as this GPU's shard:
    layout of its source ranks, all-gather of the layout counts, handle, dispatch
    of its rows into every GPU's receive buffers, a device-side barrier (a
    one-element NCCL all-reduce), the combine of its tokens reading the rows back,
    and a second barrier before the next step's dispatch overwrites any receive
    buffer.  y = the received rows (identity experts)."""

    def __init__(self, ep, w, dev, rank, world, topk_d, wts_d, x_d):
        import torch

        from combine_ep_get_11_b200 import sharded
        self.ep, self.w, self.dev, self.world = ep, w, dev, world
        R, E, T, H, K, C = w.num_ranks, w.num_experts, w.num_tokens, w.hidden, w.topk, w.num_channels
        self.r0, self.Rl = sharded.shard_ranks(R, world, rank)
        self.units = self.Rl * T
        # every token of every rank could land on each of this GPU's ranks
        cap = R * T * self.Rl
        self.buf = sharded.ShardedBuffer(R, E, T, H, K, world, rank, cap, C, device=dev)
        self.ctx = self.buf.ctx
        if world > 1:
            sharded.ProcessShardGroup(None, self.buf)        # maps the peers' buffers
        else:
            self.buf.connect({})
        self.buf.tables["y"] = list(self.buf.tables["recv_x"])    # identity experts: y = received rows
        self.out = torch.empty((self.Rl, T, H), dtype=torch.bfloat16, device=dev)
        self.out_w = torch.empty((self.Rl, T, K), dtype=torch.float32, device=dev)
        self.flag = torch.zeros(1, dtype=torch.float32, device=dev)
        self.inputs = ("x", "topk", "weights")
        self.dominant = ("dispatch", "combine")

        def device_barrier():
            if world > 1:
                import torch.distributed as dist
                dist.all_reduce(self.flag)

        def step(xd, td, wd, out=None, out_w=None):
            b = self.buf
            b.layout(td)
            if world > 1:
                import torch.distributed as dist
                dist.all_gather_into_tensor(b.ntr_all, b.ntr)
                dist.all_gather_into_tensor(b.nte_all, b.nte)
            else:
                b.ntr_all.copy_(b.ntr)
                b.nte_all.copy_(b.nte)
            b.handle()
            b.dispatch_rows(xd, td, wd)
            device_barrier()
            b.combine(self.out if out is None else out, self.out_w if out_w is None else out_w)
            device_barrier()
        self.step = step
        # one step to learn the sizes (untimed): receive rows and NVLink traffic of this GPU
        step(x_d, topk_d, wts_d)
        torch.cuda.synchronize(dev)
        ntr_all = self.buf.ntr_all.cpu().numpy()
        self.N = int(ntr_all.sum())
        self.nvlink = nvlink_traffic(ntr_all, rank, world, H, K) if world > 1 else None
        full = step_bytes(R, T, H, K, self.N, E)
        del full["step"]
        # this GPU's share of the problem's bytes (its sources' tokens and, on
        # average, its share of the receive rows)
        self.bytes = {k: v * self.Rl / R for k, v in full.items()}

    def sync_status(self):
        return self.buf.sync_status()

    def destroy(self):
        barrier(self.world)          # no shard unmaps while another still reads
        self.buf.destroy()


def time_replays(body_step, args, dev, world, flush, scrub, stream):
    """Capture the K steps once into a CUDA graph (or enqueue them eagerly) and time
    `args.repeats` replays with CUDA events on the launching stream.  Returns
    (per-replay ms, kernels this library launches per replay)."""
    import torch

    import combine_ep_get_11_b200 as ep
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(args.steps)] if flush else None

    def body():
        s = torch.cuda.current_stream(dev)
        for i in range(args.steps):
            if flush:
                scrub.sum()              # L2 flush (reads 2 x L2), outside the timed pair
                evs[i][0].record(s)
            body_step()
            if flush:
                evs[i][1].record(s)

    graph = None
    launches = 0
    if args.graph:
        launches0 = ep.kernel_launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            body()
        launches = ep.kernel_launch_count() - launches0    # kernels in one replay
    times = []
    for _ in range(args.repeats):
        barrier(world)
        torch.cuda.synchronize(dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        if args.graph:
            graph.replay()
        else:
            l0 = ep.kernel_launch_count()
            body()
            launches = ep.kernel_launch_count() - l0
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        times.append(sum(a.elapsed_time(b) for a, b in evs) if flush else ev0.elapsed_time(ev1))
    barrier(world)
    del graph
    return times, launches


def run_ours(args):
    import torch

    import combine_ep_get_11_b200 as ep

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ep.load()
    w = synth.WORKLOADS[args.workload]
    if args.tokens and args.tokens != w.num_tokens:
        w = dataclasses.replace(w.scaled(num_tokens=args.tokens), name=w.name)   # profiling runs
    sharded = args.sharded if args.sharded is not None else (world > 1 and not args.replicas)
    if sharded and w.name not in ("dsv3", "zipf", "tiny"):
        raise SystemExit("the sharded exchange runs the normal dispatch/combine workloads (dsv3, zipf, tiny)")
    if args.fp8 and w.name != "ll":
        raise SystemExit("--fp8 applies to the low-latency workload only")
    R, E, T, H, K = w.num_ranks, w.num_experts, w.num_tokens, w.hidden, w.topk

    # seeded inputs: replicas draw their own batch per rank; the sharded exchange
    # splits one problem, each GPU holding its ranks' tokens
    if sharded:
        from combine_ep_get_11_b200 import sharded as sh
        r0, Rl = sh.shard_ranks(R, world, rank)
        topk_h = torch.from_numpy(np.ascontiguousarray(synth.topk_idx(w)[r0:r0 + Rl])).pin_memory()
        wts_h = torch.from_numpy(np.ascontiguousarray(synth.topk_weights(w)[r0:r0 + Rl])).pin_memory()
        x_h = synth.hidden_rows(w, pin_memory=True, ranks=range(r0, r0 + Rl))
    else:
        ww = w if world == 1 else dataclasses.replace(w, seed=w.seed + 1000 * rank)
        topk_h = torch.from_numpy(synth.topk_idx(ww)).pin_memory()
        wts_h = torch.from_numpy(synth.topk_weights(ww)).pin_memory()
        x_h = synth.hidden_rows(ww, pin_memory=True)
    topk_d, wts_d, x_d = topk_h.to(dev), wts_h.to(dev), x_h.to(dev)
    if sharded:
        path = ShardedPath(ep, w, dev, rank, world, topk_d, wts_d, x_d)
    else:
        path = Path(ep, w, dev, topk_d, wts_d, x_d, fp8=args.fp8)
    ctx, step = path.ctx, path.step
    step_total = sum(path.bytes.values())          # this rank's bytes per step
    stream = torch.cuda.current_stream(dev)

    # inputs smaller than L2 are re-read from L2 across steps: flush between steps then
    flush = x_d.numel() * 2 < 2 * L2_BYTES and w.name != "lb"    # lb moves GB-sized expert blocks
    # flush by reading (a written scrub leaves ~L2 of dirty lines whose write-back
    # would overlap the next timed kernel)
    scrub = torch.ones(L2_BYTES, dtype=torch.float16, device=dev) if flush else None

    for _ in range(args.warmup):
        step(x_d, topk_d, wts_d)
    rc = path.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} after warm-up")
    _ = ep.ep_profile_read(ctx)
    graph_ok = args.graph and not (sharded and world > 1)    # steps with NCCL calls stay eager
    gargs = argparse.Namespace(**{**vars(args), "graph": graph_ok})

    # ---- timed region: `repeats` replays of the K steps, inputs resident in HBM.  The
    # steps run bare, as a caller runs them.  Per-kernel times come from as many
    # further replays, each of a fresh capture with the library's per-kernel events
    # (event-record nodes between the kernels, a few microseconds each).
    sampler = ClockSampler(local)
    ep.ep_profile_enable(ctx, False)
    times, launches = time_replays(lambda: step(x_d, topk_d, wts_d), gargs, dev, world, flush, scrub, stream)
    stage, prof_times = {}, []
    one = argparse.Namespace(**{**vars(gargs), "repeats": 1})
    for _ in range(args.repeats):
        ep.ep_profile_enable(ctx, True)
        t, _ = time_replays(lambda: step(x_d, topk_d, wts_d), one, dev, world, flush, scrub, stream)
        ep.ep_profile_enable(ctx, False)
        for k, (n, tot) in ep.ep_profile_read(ctx).items():
            if n:
                stage.setdefault(k, []).append(tot / n)
        prof_times += t
    clocks = sampler.stop()
    rc = path.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} after the timed region")

    per = [aggregate(t, step_total, path.units, args.steps, world, dev)[0] for t in times]
    ms_med, ms_min = statistics.median(per), min(per)
    _, gbs, tokens_per_s = aggregate(ms_med, step_total, path.units, args.steps, world, dev)
    _, gbs_best, _ = aggregate(ms_min, step_total, path.units, args.steps, world, dev)
    ms_prof = statistics.median(prof_times)

    # ---- per-kernel times (events around each launch on the call's stream)
    stage_ms = {k: statistics.median(v) for k, v in stage.items()}
    peak, peak_kind = measured_peak()
    dom = max(path.dominant, key=lambda k: stage_ms.get(k) or 0.0)
    dom_gbs = path.bytes[dom] / (stage_ms[dom] / 1e3) / 1e9
    traffic = ncu_traffic(dom) if (w.name == WORKLOAD and not args.tokens and not sharded) else None
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(dom_gbs, 1),
                "peak": peak, "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6650 GB/s",
                "traffic": traffic,
                "algorithmic_bytes_per_launch": int(path.bytes[dom]),
                "achieved_from": f"median of {len(stage[dom])} profiled replays"}
    kernels = {k: {"ms": round(stage_ms[k], 4), "ms_min": round(min(v), 4),
                   "gbs": round(path.bytes[k] / (stage_ms[k] / 1e3) / 1e9, 1) if k in path.bytes else None,
                   "gbs_best": round(path.bytes[k] / (min(v) / 1e3) / 1e9, 1) if k in path.bytes else None}
               for k, v in stage.items()}

    # ---- end to end through host buffers (pinned), same metric.  Every step copies its
    # inputs in from pinned host memory and its outputs back.  Primary number on one
    # GPU: the steps pipelined over three streams with double-buffered device inputs
    # and outputs (H2D of step i+1 and D2H of step i-1 overlap the kernels of step i);
    # the strictly serial variant is reported beside it (and is the number of a
    # sharded exchange over several GPUs).
    out_h = torch.empty(tuple(path.out.shape), dtype=torch.bfloat16, pin_memory=True)
    out_w_h = (torch.empty(tuple(path.out_w.shape), dtype=torch.float32, pin_memory=True)
               if path.out_w is not None else None)
    use_topk, use_w = "topk" in path.inputs, "weights" in path.inputs
    e2e_steps = max(3, min(args.steps, 20))

    def h2d(xd, td, wd):
        xd.copy_(x_h, non_blocking=True)
        if use_topk:
            td.copy_(topk_h, non_blocking=True)
        if use_w:
            wd.copy_(wts_h, non_blocking=True)

    def d2h(out, out_w):
        out_h.copy_(out, non_blocking=True)
        if out_w_h is not None:
            out_w_h.copy_(out_w, non_blocking=True)

    def serial(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            h2d(x_d, topk_d, wts_d)
            step(x_d, topk_d, wts_d)
            d2h(path.out, path.out_w)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    pipelined = None
    if not (sharded and world > 1):
        xb = [x_d, torch.empty_like(x_d)]
        tb = [topk_d, torch.empty_like(topk_d)]
        wb = [wts_d, torch.empty_like(wts_d)]
        ob = [path.out, torch.empty_like(path.out)]
        owb = [path.out_w, torch.empty_like(path.out_w)] if path.out_w is not None else [None, None]
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

        def pipelined(n):
            in_ready = [torch.cuda.Event(), torch.cuda.Event()]
            comp_done = [torch.cuda.Event(), torch.cuda.Event()]
            out_done = [torch.cuda.Event(), torch.cuda.Event()]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for s in (s_in, s_comp, s_out):
                s.wait_stream(stream)
            e0.record(s_in)
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(comp_done[b])       # step i-2 has consumed inputs b
                    h2d(xb[b], tb[b], wb[b])
                    in_ready[b].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(in_ready[b])
                    if i >= 2:
                        s_comp.wait_event(out_done[b])      # outputs b of step i-2 are on the host
                    step(xb[b], tb[b], wb[b], out=ob[b], out_w=owb[b])
                    comp_done[b].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[b])
                    d2h(ob[b], owb[b])
                    out_done[b].record(s_out)
            s_out.wait_stream(s_in)
            e1.record(s_out)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1)

    serial(2)
    if pipelined is not None:
        pipelined(2)
    barrier(world)
    torch.cuda.synchronize(dev)
    if pipelined is not None:
        e2e_ms, e2e_gbs, _ = aggregate(pipelined(e2e_steps), step_total, path.units, e2e_steps, world, dev)
        barrier(world)
    ser_ms, ser_gbs, _ = aggregate(serial(e2e_steps), step_total, path.units, e2e_steps, world, dev)
    if pipelined is None:
        e2e_ms, e2e_gbs = ser_ms, ser_gbs
    h2d_bytes = x_h.numel() * 2 + (topk_h.numel() * 8 if use_topk else 0) + (wts_h.numel() * 4 if use_w else 0)
    d2h_bytes = out_h.numel() * 2 + (out_w_h.numel() * 4 if out_w_h is not None else 0)
    h2d_bytes = int(sum_over_ranks(h2d_bytes, world, dev))
    d2h_bytes = int(sum_over_ranks(d2h_bytes, world, dev))

    nvlink = None
    if sharded and world > 1:
        # per GPU per step, the busier direction of the busiest GPU, over the median step time
        link = max_over_ranks(float(max(path.nvlink["send_bytes"], path.nvlink["recv_bytes"])), world, dev)
        nv_gbs = link / (ms_med / args.steps / 1e3) / 1e9
        nvlink = {"bytes_per_gpu_per_step": int(link), "achieved": round(nv_gbs, 1), "peak": NVLINK_GBS,
                  "unit": "GB/s", "frac": round(nv_gbs / NVLINK_GBS, 4),
                  "peak_source": "measured peer copy per direction per GPU (900 GB/s nominal)",
                  "counted": "dispatch rows (with ids, weights, source index) to peers plus combine reads "
                             "of rows held by peers, the busier direction"}

    cpu = check = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and w.name == WORKLOAD and not args.tokens:
        cpu = cpu_baseline(w, args.cpu_sample_tokens)
        if not sharded:
            check = combine_check(ep, path, w, x_h.view(torch.int16).numpy().view(np.uint16),
                                  topk_h.numpy(), dev)

    if rank == 0:
        if flush:
            l2 = f"L2 flushed between steps (read of {2 * L2_BYTES >> 20} MB, outside the timed pairs)"
        elif w.name == "lb":
            l2 = (f"inputs larger than L2 (expert weights {LB_EXPERTS * LB_EXPERT_ELEMS * 2 / 1e9:.2f} GB, "
                  f"replicas {LB_REPLICAS * LB_EXPERT_ELEMS * 2 / 1e9:.2f} GB > 126 MB); no flush")
        else:
            l2 = (f"inputs larger than L2 (x {R*T*H*2/1e6:.0f} MB, received rows "
                  f"{path.N*H*2/1e9:.2f} GB > 126 MB); no flush")
        mode = (f"sharded exchange over {world} GPU(s), {R // world} virtual ranks per GPU (ep_sharded_*)"
                if sharded else ("one GPU" if world == 1 else f"{world} independent replicas"))
        cfg = dict(config_dict(w, l2_note=l2), mode=mode,
                   **({"ll_packing": "fp8 e4m3, 128-channel fp32 scales"} if args.fp8 else {}))
        if w.name == "lb":   # weights, not tokens: the token fields only size the context
            cfg = {"workload": f"lb: {LB_EXPERTS} experts of {LB_EXPERT_ELEMS} bf16 (DeepSeek-V3 expert size), "
                               f"{LB_REPLICAS} redundant replicas: weight prefetch + gradient reduction",
                   "experts": LB_EXPERTS, "elems_per_expert": LB_EXPERT_ELEMS, "replicas": LB_REPLICAS,
                   "l2": l2, "mode": mode}
        line = {
            "metric": METRIC,
            "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_med / args.steps, 4),
            "higher_is_better": True, "scaling": "weak" if (world > 1 and not sharded) else "strong",
            "vs_baseline": None, "dtype": "bf16",
            "data": ("synthetic (seeded N(0,1) expert weights and gradients, seeded redundancy mapping)"
                     if w.name == "lb" else "synthetic (seeded; DeepSeek-V3-shaped routing)"),
            "tokens_per_s": None if w.name == "lb" else round(tokens_per_s, 1),
            "us_per_step": round(ms_med / args.steps * 1e3, 2),
            "timing": {"repeats": args.repeats,
                       "us_per_step": {k: round(v / args.steps * 1e3, 2) for k, v in spread(per).items()},
                       "value_best": round(gbs_best, 1),
                       "how": ("one CUDA graph of the K steps, replayed" if graph_ok else "the K steps enqueued")
                              + f" {args.repeats} times, each bracketed by CUDA events; value from the median"},
            "frac_of_peak_step": round(gbs / world / peak, 4),
            "frac_of_8tbs_step": round(gbs / world / 8000.0, 4),
            "config": cfg,
            "num_recv_rows": path.N,
            "bytes_per_step": {k: int(v) for k, v in dict(path.bytes, step=step_total).items()},
            "kernels": kernels,
            "roofline": roofline,
            "nvlink": nvlink,
            "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d_bytes,
                    "d2h_bytes_per_step": d2h_bytes, "steps": e2e_steps,
                    "ms_per_step": round(e2e_ms / e2e_steps, 3),
                    "how": ("public API, pinned host buffers, copies overlapped with the kernels "
                            "(3 streams, double-buffered)") if pipelined is not None
                    else "public API, pinned host buffers, copies and steps in one stream",
                    "serial": {"value": round(ser_gbs, 2), "ms_per_step": round(ser_ms / e2e_steps, 3)}},
            "gpu_launches": launches,
            "kernels_timed_as": ("further replays of the same K steps with the library's per-kernel "
                                 "events on the launching stream (median over the replays)"),
            "us_per_step_with_kernel_events": round(ms_prof / args.steps * 1e3, 2),
            "clocks": clocks,
            "combine_check": check,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    path.destroy()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed replays of the K steps (median and min reported)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-sample-tokens", type=int, default=CPU_SAMPLE_TOKENS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="low-latency workload: FP8 (E4M3 + scales) dispatch packing")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="enqueue the timed steps eagerly instead of replaying one CUDA graph")
    ap.add_argument("--sharded", dest="sharded", action="store_true", default=None,
                    help="run the problem's virtual ranks over the GPUs through the sharded "
                         "exchange (the default with several GPUs; on one GPU: one shard)")
    ap.add_argument("--replicas", action="store_true",
                    help="several GPUs: an independent batch per GPU instead of the sharded exchange")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default=WORKLOAD,
                    help="default dsv3 (the headline); the others are extra measurements")
    ap.add_argument("--tokens", type=int, default=0,
                    help="tokens per rank (default: the workload's 4096); smaller runs are for profiling")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    args.repeats = max(1, args.repeats)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
