"""Seeded synthetic inputs for the MoE dispatch/combine workloads.

This module only draws inputs: hidden rows, routing (top-k expert ids) and
top-k weights.  It holds none of the dispatch/combine arithmetic, and it is
the one module that both the CUDA side (tests, benchmark) and the CPU oracle
side take their inputs from.

Generator: numpy PCG64 streams, one per (workload seed, rank, stream kind),
built from ``numpy.random.SeedSequence([seed, rank, kind])``.

Workloads (shapes of DeepSeek-V3-style expert routing; all synthetic):

=========  ==  ===  =====  =====  ==  ==========================================
name        R    E      T      H   K  routing
=========  ==  ===  =====  =====  ==  ==========================================
tiny        2    8     64    256   2  K distinct experts, uniform
dsv3        8  256   4096   7168   8  K distinct uniform, each slot -1 w.p. 0.02
ll         16  256    128   7168   8  K distinct uniform; Tmax = 128
zipf       32  256   8192   7168   8  K without replacement, Zipf(s=1.2)
                                       popularity over a seeded permutation
reuse       8  256   4096   4096   8  4 distinct ranks per token, then K
                                       distinct experts among their 4*32
=========  ==  ===  =====  =====  ==  ==========================================

Hidden rows are N(0, 1) drawn in fp32 and rounded to bf16 (round to nearest
even).  Weights are a softmax (computed in fp64, stored fp32) of N(0, 1)
logits over the K slots; masked slots keep their weight.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses

import numpy as np

SEED_BASE = 0xE9000

_KIND_ROUTING = 1
_KIND_MASK = 2
_KIND_WEIGHTS = 3
_KIND_X = 4
_KIND_Y = 5
_KIND_BIAS = 6
_KIND_PERM = 7
_KIND_REDUNDANCY = 8
_KIND_CANCEL = 9
_KIND_FP8 = 10


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_ranks: int          # R
    num_experts: int        # E
    num_tokens: int         # T (per rank)
    hidden: int             # H
    topk: int               # K
    routing: str            # uniform | uniform_masked | uniform_repeats | zipf | group_limited
    seed: int
    num_channels: int = 10  # C
    max_tokens_per_rank: int = 0   # Tmax for the low-latency path (0 -> T)
    mask_prob: float = 0.0
    zipf_s: float = 1.2
    group_ranks: int = 4

    @property
    def local_experts(self) -> int:
        return self.num_experts // self.num_ranks

    @property
    def tmax(self) -> int:
        return self.max_tokens_per_rank or self.num_tokens

    def scaled(self, num_tokens: int | None = None, hidden: int | None = None,
               name: str | None = None) -> "Workload":
        return dataclasses.replace(
            self,
            num_tokens=self.num_tokens if num_tokens is None else num_tokens,
            hidden=self.hidden if hidden is None else hidden,
            max_tokens_per_rank=0 if num_tokens is not None else self.max_tokens_per_rank,
            name=name or f"{self.name}-T{num_tokens or self.num_tokens}-H{hidden or self.hidden}")


WORKLOADS = {
    "tiny": Workload("tiny", 2, 8, 64, 256, 2, "uniform", SEED_BASE + 0),
    "dsv3": Workload("dsv3", 8, 256, 4096, 7168, 8, "uniform_masked", SEED_BASE + 1,
                     mask_prob=0.02),
    "ll": Workload("ll", 16, 256, 128, 7168, 8, "uniform", SEED_BASE + 2,
                   max_tokens_per_rank=128),
    "zipf": Workload("zipf", 32, 256, 8192, 7168, 8, "zipf", SEED_BASE + 3),
    "reuse": Workload("reuse", 8, 256, 4096, 4096, 8, "group_limited", SEED_BASE + 4),
    # redundant-expert load balance (weights, not tokens: the token fields size the
    # context only)
    "lb": Workload("lb", 8, 256, 16, 128, 8, "uniform", SEED_BASE + 5),
}


def _rng(seed: int, rank: int, kind: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, rank, kind])))


def _distinct_uniform(rng, T, n, K):
    """K distinct values of range(n) per row, uniformly at random, in draw order."""
    keys = rng.random((T, n))
    return np.argsort(keys, axis=1, kind="stable")[:, :K]


def _zipf_weights(E, s):
    ranks = np.arange(1, E + 1, dtype=np.float64)
    p = ranks ** (-s)
    return p / p.sum()


def topk_idx(w: Workload) -> np.ndarray:
    """[R, T, K] int64 expert ids (-1 = unused slot)."""
    R, E, T, K = w.num_ranks, w.num_experts, w.num_tokens, w.topk
    out = np.empty((R, T, K), np.int64)
    if w.routing == "zipf":
        perm = _rng(w.seed, 0, _KIND_PERM).permutation(E)
        p = _zipf_weights(E, w.zipf_s)
        logp = np.empty(E)
        logp[perm] = np.log(p)          # expert perm[i] has popularity rank i+1
    for s in range(R):
        rng = _rng(w.seed, s, _KIND_ROUTING)
        if w.routing in ("uniform", "uniform_masked"):
            out[s] = _distinct_uniform(rng, T, E, K)
        elif w.routing == "uniform_repeats":
            # K independent uniform draws: a token may name an expert twice
            out[s] = rng.integers(0, E, (T, K))
        elif w.routing == "zipf":
            # Sequential draws without replacement, each proportional to the
            # remaining popularity mass, are the top-K of log p + Gumbel noise.
            g = -np.log(-np.log(rng.random((T, E))))
            out[s] = np.argsort(-(logp[None, :] + g), axis=1, kind="stable")[:, :K]
        elif w.routing == "group_limited":
            L = w.local_experts
            ranks = _distinct_uniform(rng, T, w.num_ranks, w.group_ranks)          # [T, G]
            cand = (ranks[:, :, None] * L + np.arange(L)[None, None, :]).reshape(T, -1)
            pick = _distinct_uniform(rng, T, cand.shape[1], K)
            out[s] = np.take_along_axis(cand, pick, axis=1)
        else:
            raise ValueError(w.routing)
        if w.mask_prob > 0:
            m = _rng(w.seed, s, _KIND_MASK).random((T, K)) < w.mask_prob
            out[s][m] = -1
    return out


def topk_weights(w: Workload) -> np.ndarray:
    """[R, T, K] float32 softmax weights."""
    R, T, K = w.num_ranks, w.num_tokens, w.topk
    out = np.empty((R, T, K), np.float32)
    for s in range(R):
        logits = _rng(w.seed, s, _KIND_WEIGHTS).standard_normal((T, K))
        z = np.exp(logits - logits.max(axis=1, keepdims=True))
        out[s] = (z / z.sum(axis=1, keepdims=True)).astype(np.float32)
    return out


def _normal_bf16_rows(seed, kind, shape_per_rank, num_parts, torch_out):
    """Fill torch_out[part] (bf16) with N(0,1) fp32 draws rounded to bf16."""
    import torch

    def one(part):
        a = _rng(seed, part, kind).standard_normal(shape_per_rank, dtype=np.float32)
        torch_out[part].copy_(torch.from_numpy(a).to(torch.bfloat16))

    workers = min(8, max(1, num_parts))
    with _cf.ThreadPoolExecutor(workers) as ex:
        list(ex.map(one, range(num_parts)))
    return torch_out


def hidden_rows(w: Workload, pin_memory: bool = False, ranks=None):
    """x [R, T, H] torch.bfloat16 on the CPU (ranks: a range of source ranks, whose
    rows are drawn alone: [len(ranks), T, H], the same values as in the full x)."""
    import torch
    ranks = range(w.num_ranks) if ranks is None else ranks
    x = torch.empty((len(ranks), w.num_tokens, w.hidden), dtype=torch.bfloat16, pin_memory=pin_memory)

    def one(i):
        a = _rng(w.seed, ranks[i], _KIND_X).standard_normal((w.num_tokens, w.hidden), dtype=np.float32)
        x[i].copy_(torch.from_numpy(a).to(torch.bfloat16))

    with _cf.ThreadPoolExecutor(min(8, max(1, len(ranks)))) as ex:
        list(ex.map(one, range(len(ranks))))
    return x


def expert_rows(seed: int, num_rows: int, hidden: int, chunk: int = 65536):
    """An independent N(0,1) bf16 tensor [num_rows, H] (stand-in expert outputs)."""
    import torch
    y = torch.empty((num_rows, hidden), dtype=torch.bfloat16)
    parts = (num_rows + chunk - 1) // chunk

    def one(part):
        lo, hi = part * chunk, min(num_rows, (part + 1) * chunk)
        a = _rng(seed, part, _KIND_Y).standard_normal((hi - lo, hidden), dtype=np.float32)
        y[lo:hi].copy_(torch.from_numpy(a).to(torch.bfloat16))

    with _cf.ThreadPoolExecutor(min(8, max(1, parts))) as ex:
        list(ex.map(one, range(parts)))
    return y


def cancel_rows(seed: int, num_rows: int, hidden: int, p_big: float = 0.5, big_exp: int = 25):
    """[num_rows, H] numpy uint16 bf16 bit patterns whose sums cancel: each value
    is +-2^big_exp (random sign) with probability p_big, else an N(0,1) draw
    rounded to bf16.  Where the large terms of a sum cancel, the small ones that
    were added next to a large one lost their low bits (binary32 keeps 24
    significant bits), so the result depends on the order of the additions.
    N(0,1) rows seldom show the order: their sums of a few terms are mostly
    exact in binary32."""
    import torch
    rng = _rng(seed, 0, _KIND_CANCEL)
    big = rng.random((num_rows, hidden)) < p_big
    sign = np.where(rng.random((num_rows, hidden)) < 0.5, -1.0, 1.0)
    small = rng.standard_normal((num_rows, hidden), dtype=np.float32)
    v = np.where(big, sign * 2.0 ** big_exp, small).astype(np.float32)
    return torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def cancel_rows_device(seed: int, num_rows: int, hidden: int, device="cuda", p_big: float = 0.5,
                       big_exp: int = 25, chunk_rows: int = 1 << 16):
    """cancel_rows' distribution drawn on the GPU with torch's seeded generator (bf16
    tensor [num_rows, H]) for full-size workloads."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    y = torch.empty((num_rows, hidden), dtype=torch.bfloat16, device=device)
    for lo in range(0, num_rows, chunk_rows):
        hi = min(num_rows, lo + chunk_rows)
        shape = (hi - lo, hidden)
        big = torch.rand(shape, generator=gen, device=device) < p_big
        sign = torch.where(torch.rand(shape, generator=gen, device=device) < 0.5, -1.0, 1.0)
        small = torch.randn(shape, generator=gen, device=device)
        y[lo:hi] = torch.where(big, sign * float(2 ** big_exp), small)
    return y


def fp8_block_rows(seed: int, num_rows: int, hidden: int, block: int = 128):
    """[num_rows, H] numpy uint16 bf16 bit patterns whose 128-channel blocks take
    the cases an FP8 block quantiser must get right, one kind per block in turn:
    all +0; all -0; signed zeros with a single +1 or -1; a negative largest
    magnitude among small positives; N(0,1) x 2^124; N(0,1) x 2^-100 (the
    block's 448 / amax still finite); E4M3 rounding ties (amax 448, so the
    products are the values themselves: halfway points between E4M3 neighbours,
    normal and subnormal); N(0,1) with a few bf16 subnormals."""
    rng = _rng(seed, 0, _KIND_FP8)
    nb = hidden // block
    v = np.zeros((num_rows, hidden), dtype=np.float32)
    # halfway points between adjacent E4M3 values (exact in bf16: 5 significant bits)
    ties = np.array([1.0625, 1.1875, 3.25 + 0.125, 2.0 ** -7 + 2.0 ** -10, 2.0 ** -9 * 1.5,
                     2.0 ** -9 * 0.5, 240.0 + 8.0, 416.0 + 16.0], dtype=np.float32)
    for r in range(num_rows):
        for b in range(nb):
            kind = (r * nb + b) % 8
            blk = v[r, b * block:(b + 1) * block]
            if kind == 1:
                blk[:] = -0.0
            elif kind == 2:
                blk[:] = np.where(rng.random(block) < 0.5, -0.0, 0.0)
                blk[rng.integers(block)] = 1.0 if rng.random() < 0.5 else -1.0
            elif kind == 3:
                blk[:] = rng.random(block) * 0.5
                blk[rng.integers(block)] = -3.5
            elif kind == 4:
                blk[:] = rng.standard_normal(block) * 2.0 ** 124
            elif kind == 5:
                blk[:] = rng.standard_normal(block) * 2.0 ** -100
            elif kind == 6:
                blk[:] = rng.choice(ties, block) * np.where(rng.random(block) < 0.5, -1.0, 1.0)
                blk[rng.integers(block)] = 448.0
            elif kind == 7:
                blk[:] = rng.standard_normal(block)
                blk[rng.integers(block, size=4)] = 2.0 ** -130
    import torch
    return torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bias_rows(w: Workload, which: int):
    """bias tensor [R, T, H] bf16, N(0,1)."""
    import torch
    b = torch.empty((w.num_ranks, w.num_tokens, w.hidden), dtype=torch.bfloat16)
    return _normal_bf16_rows(w.seed + 7919 * (which + 1), _KIND_BIAS,
                             (w.num_tokens, w.hidden), w.num_ranks, b)


def expert_rows_device(seed: int, num_rows: int, hidden: int, device="cuda", chunk_rows: int = 1 << 16):
    """An independent N(0,1) bf16 tensor [num_rows, H] drawn on the GPU with torch's
    seeded generator (for full-size workloads whose expert outputs are too large to
    draw on the host).  Deterministic for a given seed, device type and torch build."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    y = torch.empty((num_rows, hidden), dtype=torch.bfloat16, device=device)
    for lo in range(0, num_rows, chunk_rows):
        hi = min(num_rows, lo + chunk_rows)
        y[lo:hi] = torch.randn((hi - lo, hidden), generator=gen, device=device, dtype=torch.float32)
    return y


def redundancy_mapping(num_experts: int, num_redundant: int, seed: int, unused_prob: float = 0.0):
    """[N] int32: the original expert of each redundant replica (seeded; an expert may have
    several replicas; -1 marks an unused replica slot with probability unused_prob)."""
    rng = _rng(seed, 0, _KIND_REDUNDANCY)
    m = rng.integers(0, num_experts, num_redundant).astype(np.int32)
    if unused_prob > 0:
        m[rng.random(num_redundant) < unused_prob] = -1
    return m
