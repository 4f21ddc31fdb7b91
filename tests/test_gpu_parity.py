"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by
element, on seeded inputs small enough for the oracle, spanning several scan tiles,
several dispatch CTAs and ragged tails.  Everything is bit-exact: integer, index and
copied-row outputs, and the combines against the oracle's fixed-order fp32
definition (ascending ranks / expert ids, binary32, one bf16 rounding).  Rows whose
large terms cancel make the summation order visible; against the exact sums the
combines are also checked within one bf16 ulp (N(0,1) rows) or the binary32
summation bound (cancelling rows), and the error statistics are reported."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import Inputs, bf16_abs, check_combine, load_golden_fp32, to_bf16_tensor, u16

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = [
    W["tiny"],
    W["dsv3"].scaled(num_tokens=300),                    # 2400 tokens, H = 7168
    W["ll"].scaled(num_tokens=77, hidden=1024),
    W["zipf"].scaled(num_tokens=70, hidden=512),         # 32 ranks, skewed destinations
    W["reuse"].scaled(num_tokens=260),                   # H = 4096, group-limited
    synth.Workload("odd", 3, 9, 50, 24, 4, "uniform", 99, num_channels=7),
    synth.Workload("top1", 4, 8, 33, 64, 1, "uniform_masked", 98, num_channels=3, mask_prob=0.3),
    synth.Workload("one-rank", 1, 6, 40, 16, 2, "uniform_masked", 97, num_channels=4, mask_prob=0.3),
    synth.Workload("chan>T", 2, 4, 5, 8, 2, "uniform", 96, num_channels=12),
    # limits: 32 ranks with top-32 (fan-out up to 32), the widest row, the narrowest row,
    # the most experts
    synth.Workload("R32-K32", 32, 64, 40, 64, 32, "uniform", 89, num_channels=5),
    synth.Workload("H32768", 2, 4, 20, 32768, 2, "uniform", 88, num_channels=3),
    synth.Workload("H8", 2, 4, 33, 8, 2, "uniform_masked", 87, num_channels=2, mask_prob=0.2),
    synth.Workload("E4096", 8, 4096, 50, 16, 8, "uniform", 86, num_channels=4),
    # a token may name an expert twice (counted twice per expert, once per rank)
    synth.Workload("repeats", 4, 16, 70, 64, 5, "uniform_repeats", 76, num_channels=3, mask_prob=0.1),
    # more tokens per source than one layout cluster covers in one pass (8 CTAs of 512
    # threads): each CTA walks two token blocks, the last one ragged
    synth.Workload("layout-2pass", 3, 12, 4700, 32, 4, "uniform_masked", 75, num_channels=6, mask_prob=0.1),
]


def ids(ws):
    return [w.name for w in ws]


@pytest.fixture(scope="module")
def ep(cuda_lib):
    return cuda_lib


def make_buffer(ep, w):
    return ep.Buffer(w.num_ranks, w.num_experts, w.num_tokens, w.hidden, w.topk, w.num_channels,
                     w.max_tokens_per_rank)


def oracle_normal(inp):
    w = inp.w
    ntr, nte, tin = oracle.layout(inp.topk, w.num_experts)
    h = oracle.dispatch_handle(tin, nte, w.num_channels)
    rows = oracle.dispatch_rows(inp.x_u16, inp.topk, inp.weights, h, w.num_experts)
    return (ntr, nte, tin), h, rows


HANDLE_KEYS = ("rank_prefix_matrix", "channel_prefix_matrix", "recv_channel_prefix_matrix",
               "send_head", "recv_rank_offset", "num_recv_tokens_per_expert", "is_token_in_rank")


@pytest.mark.parametrize("w", CASES, ids=ids(CASES))
def test_layout_handle_dispatch_combine(ep, w):
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    (ntr, nte, tin), h, (o_recv_x, o_idx, o_w) = oracle_normal(inp)
    N = int(h["recv_rank_offset"][-1])

    layout = buf.get_dispatch_layout(inp.topk_d)
    for got, exp, name in zip(layout, (ntr, nte, tin), ("ntr", "nte", "is_token_in_rank")):
        np.testing.assert_array_equal(got.cpu().numpy(), exp, err_msg=name)
    n_all, n_per = ep.ep_get_num_recv(buf.ctx, layout[0], w.num_ranks)
    assert n_all == N and n_per == np.diff(h["recv_rank_offset"]).tolist()

    recv_x, recv_idx, recv_w, handle = buf.dispatch(inp.x_d, inp.topk_d, inp.weights_d, layout=layout)
    assert buf.sync_status() == 0
    assert handle.num_recv_rows == N
    for key in HANDLE_KEYS:
        np.testing.assert_array_equal(getattr(handle, key).cpu().numpy(), h[key], err_msg=key)
    np.testing.assert_array_equal(handle.recv_src_idx.cpu().numpy()[:N], h["recv_src_idx"])
    np.testing.assert_array_equal(u16(recv_x), o_recv_x)
    np.testing.assert_array_equal(recv_idx.cpu().numpy(), o_idx)
    np.testing.assert_array_equal(recv_w.cpu().numpy(), o_w)

    # identity experts: every sum is exact, so the combine is bit-exact
    out, out_w = buf.combine(recv_x, handle, recv_w)
    e_out, e_w = oracle.combine(o_recv_x, h, o_w)
    np.testing.assert_array_equal(u16(out), e_out)
    np.testing.assert_array_equal(out_w.cpu().numpy(), e_w)

    # independent expert outputs and two bias terms
    y = synth.expert_rows(w.seed + 1, N, w.hidden)
    b0, b1 = synth.bias_rows(w, 0), synth.bias_rows(w, 1)
    out2, _ = buf.combine(y.cuda(), handle, None, bias=(b0.cuda(), b1.cuda()))
    bias = dict(bias0=u16(b0), bias1=u16(b1))
    check_combine(f"{w.name}: combine, N(0,1) rows + 2 biases", u16(out2),
                  oracle.combine(u16(y), h, fp32=True, **bias)[0], oracle.combine(u16(y), h, **bias)[0],
                  one_ulp=True)
    # rows whose large terms cancel (the order of the additions shows), and received
    # weight rows that cancel too (the weights' sum order shows)
    yc = synth.cancel_rows(w.seed + 2, N, w.hidden)
    wc = synth.cancel_rows(w.seed + 3, N, w.topk)
    wc = ((wc.astype(np.uint32) << 16).view(np.float32)).copy()
    out3, out3_w = buf.combine(to_bf16_tensor(yc).cuda(), handle, torch.from_numpy(wc).cuda())
    ref32, ref32_w = oracle.combine(yc, h, wc, fp32=True)
    exact, _ = oracle.combine(yc, h, wc)
    abs_sum, _ = oracle.combine(bf16_abs(yc), h)
    check_combine(f"{w.name}: combine, cancelling rows", u16(out3), ref32, exact, abs_sum,
                  min(w.num_ranks, w.topk), cancelling=True)
    np.testing.assert_array_equal(out3_w.cpu().numpy(), ref32_w, err_msg="combined weights, fixed order")

    # cached dispatch of new rows with the same handle
    x2 = synth.hidden_rows(dataclasses.replace(w, seed=w.seed + 17))
    recv_x2 = buf.dispatch_cached(x2.cuda(), handle)
    e_x2, _, _ = oracle.dispatch_rows(u16(x2), inp.topk, None, h, w.num_experts)
    np.testing.assert_array_equal(u16(recv_x2), e_x2)
    assert buf.sync_status() == 0
    buf.destroy()


def test_hand_worked_fp32_cases(ep):
    """The hand-worked cancellation cases of tests/golden/fp32_order.txt through the C
    ABI: the combine adds in ascending rank order with the biases last, the
    low-latency combine is a fused multiply-add chain over ascending expert ids, the
    gradient reduction adds replicas in ascending order.  The fixtures' columns come
    first in rows of 8 (whole 16-byte vectors); the other columns are zero."""
    g = load_golden_fp32()
    H = 8

    def rows(bits, n, width):
        a = np.zeros((n, H), np.uint16)
        a[:, :width] = np.array(bits, np.uint16).reshape(n, width)
        return a

    # combine: token (0, 0) of three ranks names experts 0, 1, 2 (one per rank)
    R, T, K, hc = g["combine_R"][0], g["combine_T"][0], 3, g["combine_H"][0]
    buf = ep.Buffer(R, R, T, H, K, 1)
    topk = torch.tensor([[[0, 1, 2]], [[-1, -1, -1]], [[-1, -1, -1]]], dtype=torch.int64, device="cuda")
    x = torch.zeros((R, T, H), dtype=torch.bfloat16, device="cuda")
    _, _, _, handle = buf.dispatch(x, topk)
    assert handle.send_head.cpu().numpy().ravel().tolist() == g["combine_send_head"]
    assert handle.recv_rank_offset.cpu().numpy().tolist() == g["combine_recv_rank_offset"]
    y = to_bf16_tensor(rows(g["combine_y"], 3, hc)).cuda()
    b0 = to_bf16_tensor(rows(g["combine_bias0"], R * T, hc).reshape(R, T, H)).cuda()
    b1 = to_bf16_tensor(rows(g["combine_bias1"], R * T, hc).reshape(R, T, H)).cuda()
    rw = np.zeros((3, K), np.float32)
    rw[:, 0] = np.array(g["combine_recv_w"], np.uint32).view(np.float32)
    out, out_w = buf.combine(y, handle, torch.from_numpy(rw).cuda(), bias=(b0, b1))
    assert buf.sync_status() == 0
    got = u16(out).reshape(R * T, H)
    assert got[:, :hc].ravel().tolist() == g["combine_out_fp32"]
    assert not got[:, hc:].any()
    ow = out_w.cpu().numpy().reshape(R * T, K)
    assert ow[:, 0].view(np.uint32).tolist() == g["combine_w_fp32"]
    assert not ow[:, 1:].any()
    buf.destroy()

    # low-latency combine
    R, E, T, K, Tmax = (g[f"ll_{k}"][0] for k in ("R", "E", "T", "K", "TMAX"))
    buf = ep.Buffer(R, E, T, H, K, 1, Tmax)
    topk = torch.tensor(g["ll_topk_idx"], dtype=torch.int64).reshape(R, T, K).cuda()
    _, count, ll_handle = buf.low_latency_dispatch(torch.zeros((R, T, H), dtype=torch.bfloat16,
                                                               device="cuda"), topk)
    assert count.cpu().numpy().ravel().tolist() == [1, 2, 1, 1]
    y = to_bf16_tensor(rows(g["ll_y"], E * R * Tmax, 1).reshape(R, E // R, R * Tmax, H)).cuda()
    wts = torch.from_numpy(np.array(g["ll_w"], np.uint32).view(np.float32).reshape(R, T, K)).cuda()
    out = buf.low_latency_combine(y, topk, wts, ll_handle)
    assert buf.sync_status() == 0
    got = u16(out).reshape(R * T, H)
    assert got[:, 0].tolist() == g["ll_out_fp32"]
    assert not got[:, 1:].any()
    buf.destroy()

    # gradient reduction: one expert, two replicas
    buf = ep.Buffer(1, 1, 1, H, 1, 1)
    grads = to_bf16_tensor(rows(g["lb_grads"], 1, 1)).cuda()
    red = to_bf16_tensor(rows(g["lb_redundant"], 2, 1)).cuda()
    buf.lb_reduce_grads(red, grads, torch.tensor(g["lb_mapping"], dtype=torch.int32, device="cuda"))
    assert buf.sync_status() == 0
    got = u16(grads)
    assert got[:, 0].tolist() == g["lb_out_fp32"]
    assert not got[:, 1:].any()
    buf.destroy()


@pytest.mark.parametrize("w", CASES[:5], ids=ids(CASES[:5]))
def test_dispatch_computes_layout_itself(ep, w):
    """ep_dispatch without a precomputed layout builds the same handle and rows."""
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    _, h, (o_recv_x, _, _) = oracle_normal(inp)
    N = int(h["recv_rank_offset"][-1])
    handle = ep.Handle.empty(w.num_ranks, w.num_tokens, w.num_channels, w.local_experts, N, "cuda")
    recv_x = torch.empty((N, w.hidden), dtype=torch.bfloat16, device="cuda")
    n = ep.ep_dispatch(buf.ctx, inp.x_d, inp.topk_d, None, None, None, None, handle, recv_x, None,
                       None, N, want_num_recv=True)
    assert n == N
    for key in HANDLE_KEYS:
        np.testing.assert_array_equal(getattr(handle, key).cpu().numpy(), h[key], err_msg=key)
    np.testing.assert_array_equal(u16(recv_x), o_recv_x)
    assert buf.sync_status() == 0
    buf.destroy()


LL_CASES = [
    W["ll"].scaled(num_tokens=40, hidden=1024),
    W["tiny"],
    dataclasses.replace(W["ll"].scaled(num_tokens=50, hidden=256), max_tokens_per_rank=64,
                        name="ll-tmax64"),
    synth.Workload("ll-odd", 3, 12, 30, 40, 5, "uniform_masked", 95, mask_prob=0.2),
    # more than two 2048-token chunks of the slot kernel, 32 ranks
    synth.Workload("ll-big", 32, 256, 160, 64, 8, "uniform", 94),
    synth.Workload("ll-k20", 4, 64, 50, 32, 20, "uniform_masked", 93, mask_prob=0.1),
    synth.Workload("ll-E4096", 8, 4096, 40, 128, 8, "uniform", 92),
    # sources longer than one 256-token slot tile (3 tiles each, the last one ragged):
    # the lookback scan; at most 256 tokens per source: direct slots
    synth.Workload("ll-T600", 4, 32, 600, 64, 4, "uniform_masked", 91, mask_prob=0.1),
    synth.Workload("ll-T256", 4, 32, 256, 128, 8, "uniform_masked", 79, mask_prob=0.05),
    synth.Workload("ll-T257", 4, 32, 257, 128, 8, "uniform_masked", 78, mask_prob=0.05),
    # repeated experts within a token (a token counts once per expert)
    synth.Workload("ll-rep-experts", 4, 8, 90, 128, 6, "uniform_repeats", 77, mask_prob=0.1),
    # the widest row (FP8: 64 steps of 512 channels, 32 slices per token)
    synth.Workload("ll-H32768", 2, 4, 12, 32768, 2, "uniform", 73),
]


@pytest.mark.parametrize("w", LL_CASES, ids=ids(LL_CASES))
def test_low_latency(ep, w):
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    packed, count, (src_info, layout_range) = buf.low_latency_dispatch(inp.x_d, inp.topk_d)
    assert buf.sync_status() == 0
    ll = oracle.ll_dispatch(inp.x_u16, inp.topk, w.num_experts, w.tmax)
    np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
    np.testing.assert_array_equal(layout_range.cpu().numpy(), ll["layout_range"])
    p = u16(packed)
    si = src_info.cpu().numpy()
    R, L = w.num_ranks, w.local_experts
    for d in range(R):
        for j in range(L):
            n = int(ll["packed_recv_count"][d, j])
            np.testing.assert_array_equal(si[d, j, :n], ll["src_info"][d, j, :n])
            np.testing.assert_array_equal(p[d, j, :n], ll["packed_recv_x"][d, j, :n])
    # identity experts and independent expert outputs (softmax weights), then rows
    # whose large terms cancel with unit weights (the order of the chain shows)
    rows = R * L * w.tmax * w.num_ranks
    ones = np.ones_like(inp.weights)
    for what, y_u16, wts in (
            ("identity experts", p, inp.weights),
            ("N(0,1) rows", u16(synth.expert_rows(w.seed + 3, rows, w.hidden)).reshape(p.shape), inp.weights),
            ("cancelling rows, unit weights", synth.cancel_rows(w.seed + 4, rows, w.hidden).reshape(p.shape),
             ones)):
        y_d = to_bf16_tensor(y_u16).cuda()
        out = buf.low_latency_combine(y_d, inp.topk_d, torch.from_numpy(wts).cuda(), (src_info, layout_range))
        args = (ll["src_info"], ll["layout_range"], w.num_experts, w.tmax)
        ref32 = oracle.ll_combine(y_u16, inp.topk, wts, *args, fp32=True)
        exact = oracle.ll_combine(y_u16, inp.topk, wts, *args)
        abs_ref = oracle.ll_combine(bf16_abs(y_u16), inp.topk, np.abs(wts), *args)
        check_combine(f"{w.name}: ll combine, {what}", u16(out), ref32, exact, abs_ref, w.topk,
                      cancelling=what.startswith("cancelling"))
    assert buf.sync_status() == 0
    buf.destroy()


# ----------------------------------------------------------------------------- repeated calls

def test_repeated_calls_on_one_context(ep):
    """The scans keep their status words between calls (tagged with the call): calls
    with other routings on the same context must not see a previous call's words."""
    base = W["dsv3"].scaled(num_tokens=700, hidden=64)           # 5600 tokens: 22 scan tiles
    buf = make_buffer(ep, base)
    for seed in (base.seed, base.seed + 1, base.seed, base.seed + 2):
        w = dataclasses.replace(base, seed=seed)
        inp = Inputs(w)
        _, h, (o_recv_x, _, _) = oracle_normal(inp)
        recv_x, _, _, handle = buf.dispatch(inp.x_d, inp.topk_d, inp.weights_d)
        for key in HANDLE_KEYS:
            np.testing.assert_array_equal(getattr(handle, key).cpu().numpy(), h[key], err_msg=key)
        np.testing.assert_array_equal(u16(recv_x), o_recv_x)
    assert buf.sync_status() == 0
    buf.destroy()

    # low-latency slots: the lookback scan (300 tokens per source) and the direct
    # slots (200 tokens per source: per-source counts and ranks rewritten by every
    # call, with routings that change between calls)
    for base in (synth.Workload("ll-rep", 8, 64, 300, 64, 6, "uniform_masked", 84, mask_prob=0.1),
                 synth.Workload("ll-rep-direct", 8, 64, 200, 64, 6, "uniform_masked", 85, mask_prob=0.1)):
        buf = make_buffer(ep, base)
        for seed in (base.seed, base.seed + 1, base.seed, base.seed + 2):
            w = dataclasses.replace(base, seed=seed)
            inp = Inputs(w)
            packed, count, (src_info, layout_range) = buf.low_latency_dispatch(inp.x_d, inp.topk_d)
            ll = oracle.ll_dispatch(inp.x_u16, inp.topk, w.num_experts, w.tmax)
            np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
            np.testing.assert_array_equal(layout_range.cpu().numpy(), ll["layout_range"])
            si, pk = src_info.cpu().numpy(), u16(packed)
            for d in range(w.num_ranks):
                for j in range(w.local_experts):
                    n = int(ll["packed_recv_count"][d, j])
                    np.testing.assert_array_equal(si[d, j, :n], ll["src_info"][d, j, :n])
                    np.testing.assert_array_equal(pk[d, j, :n], ll["packed_recv_x"][d, j, :n])
        assert buf.sync_status() == 0
        buf.destroy()


def test_ll_combine_with_an_older_handle(ep):
    """The low-latency combine takes the last dispatch's slots only where the
    handle it is given confirms them: combining routing A's rows with A's handle
    after a dispatch of routing B must still give A's result."""
    w = synth.Workload("ll-old", 8, 64, 96, 128, 6, "uniform_masked", 80, mask_prob=0.1)
    a = Inputs(w)
    b = Inputs(dataclasses.replace(w, seed=w.seed + 1))
    buf = make_buffer(ep, w)
    packed_a, _, handle_a = buf.low_latency_dispatch(a.x_d, a.topk_d)
    buf.low_latency_dispatch(b.x_d, b.topk_d)                     # the context now holds B's slots
    out = buf.low_latency_combine(packed_a, a.topk_d, a.weights_d, handle_a)
    assert buf.sync_status() == 0
    ll = oracle.ll_dispatch(a.x_u16, a.topk, w.num_experts, w.tmax)
    args = (ll["src_info"], ll["layout_range"], w.num_experts, w.tmax)
    check_combine("ll combine with an older handle", u16(out),
                  oracle.ll_combine(ll["packed_recv_x"], a.topk, a.weights, *args, fp32=True),
                  oracle.ll_combine(ll["packed_recv_x"], a.topk, a.weights, *args),
                  oracle.ll_combine(bf16_abs(ll["packed_recv_x"]), a.topk, np.abs(a.weights), *args), w.topk)
    buf.destroy()


def test_handle_check(ep):
    """The reuse contract: a handle checks out against its own routing, or one that
    sends every token to the same ranks, and fails against any other."""
    w = W["dsv3"].scaled(num_tokens=300, hidden=64)
    a = Inputs(w)
    b = Inputs(dataclasses.replace(w, seed=w.seed + 1))
    buf = make_buffer(ep, w)
    _, _, _, handle = buf.dispatch(a.x_d, a.topk_d, a.weights_d)
    assert buf.check_handle(a.topk_d, handle)
    assert not buf.check_handle(b.topk_d, handle)
    L = w.local_experts
    topk = a.topk.copy()
    flat = topk.reshape(-1, w.topk)
    # same ranks: swap one expert for another expert of the same rank
    g = int(np.nonzero(flat[:, 0] >= 0)[0][0])
    e = int(flat[g, 0])
    flat[g, 0] = e // L * L + (e % L + 1) % L
    assert buf.check_handle(torch.from_numpy(topk).cuda(), handle)
    # another rank: one token's set of destination ranks changes
    for g in range(flat.shape[0]):
        ranks = {int(x) // L for x in flat[g] if x >= 0}
        if len(ranks) < w.num_ranks and flat[g, 0] >= 0:
            break
    r = next(r for r in range(w.num_ranks) if r not in ranks)
    flat[g, 0] = r * L
    assert not buf.check_handle(torch.from_numpy(topk).cuda(), handle)
    assert buf.sync_status() == 0
    buf.destroy()


# ----------------------------------------------------------------------------- bounded waits

def test_bounded_wait_runs_out_and_context_recovers(ep):
    """Failure detection without a fault: shift the scans' ticket counters by one,
    so the next scan's tiles carry two different call tags and the tiles waiting
    for a word tagged with the other number give up after the wait limit.  The
    call must end (no hang), report EP_ERR_TIMEOUT, and the context must give
    correct results afterwards (ep_sync_status realigns the counters)."""
    import time
    w = synth.Workload("wait", 4, 16, 300, 64, 4, "uniform", 81)   # 5 handle tiles, 8 slot tiles
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    ll = oracle.ll_dispatch(inp.x_u16, inp.topk, w.num_experts, w.tmax)
    _, h, (o_recv_x, _, _) = oracle_normal(inp)
    N = int(h["recv_rank_offset"][-1])
    handle = ep.Handle.empty(w.num_ranks, w.num_tokens, w.num_channels, w.local_experts, N, "cuda")
    recv_x = torch.empty((N, w.hidden), dtype=torch.bfloat16, device="cuda")

    def dispatch():
        ep.ep_dispatch(buf.ctx, inp.x_d, inp.topk_d, None, None, None, None, handle, recv_x, None, None, N)

    def check_ll():
        _, count, (src_info, layout_range) = buf.low_latency_dispatch(inp.x_d, inp.topk_d)
        assert buf.sync_status() == 0
        np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
        np.testing.assert_array_equal(layout_range.cpu().numpy(), ll["layout_range"])

    def check_normal():
        dispatch()
        assert buf.sync_status() == 0
        for key in ("send_head", "rank_prefix_matrix", "channel_prefix_matrix", "recv_rank_offset"):
            np.testing.assert_array_equal(getattr(handle, key).cpu().numpy(), h[key], err_msg=key)
        np.testing.assert_array_equal(u16(recv_x), o_recv_x)

    check_ll()
    check_normal()
    lib = ep.load()
    for skewed in (lambda: buf.low_latency_dispatch(inp.x_d, inp.topk_d), dispatch):
        assert lib.ep_test_offset_tickets(buf.ctx, 1) == 0
        t0 = time.monotonic()
        skewed()                              # outputs undefined: some tiles give up
        assert buf.sync_status() == 6         # EP_ERR_TIMEOUT
        assert time.monotonic() - t0 < 60
        check_ll()
        check_normal()
    buf.destroy()


# ----------------------------------------------------------------------------- edge cases

def test_no_tokens(ep):
    w = synth.Workload("empty", 4, 16, 0, 64, 2, "uniform", 1)
    buf = make_buffer(ep, w)
    topk = torch.empty((4, 0, 2), dtype=torch.int64, device="cuda")
    x = torch.empty((4, 0, 64), dtype=torch.bfloat16, device="cuda")
    recv_x, recv_idx, _, handle = buf.dispatch(x, topk)
    assert recv_x.shape[0] == 0
    assert handle.recv_rank_offset.cpu().tolist() == [0] * 5
    ntr, _, _ = buf.get_dispatch_layout(topk)
    assert ep.ep_get_num_recv(buf.ctx, ntr, 4) == (0, [0, 0, 0, 0])
    assert not handle.rank_prefix_matrix.any() and not handle.channel_prefix_matrix.any()
    out, _ = buf.combine(recv_x, handle)
    assert out.numel() == 0
    assert buf.sync_status() == 0
    buf.destroy()


def test_all_slots_masked(ep):
    w = synth.Workload("masked", 2, 8, 100, 64, 2, "uniform", 2)
    buf = make_buffer(ep, w)
    topk = torch.full((2, 100, 2), -1, dtype=torch.int64, device="cuda")
    x = torch.randn((2, 100, 64), device="cuda").to(torch.bfloat16)
    ntr, _, _ = buf.get_dispatch_layout(topk)
    assert ep.ep_get_num_recv(buf.ctx, ntr, 2) == (0, [0, 0])
    recv_x, _, _, handle = buf.dispatch(x, topk)
    assert recv_x.shape[0] == 0
    assert (handle.send_head == -1).all()
    out, _ = buf.combine(recv_x, handle)
    assert (out == 0).all()
    assert buf.sync_status() == 0
    buf.destroy()


def test_capacity_overflow_is_reported_not_written(ep):
    w = W["tiny"]
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    _, h, (o_recv_x, _, _) = oracle_normal(inp)
    N = int(h["recv_rank_offset"][-1])
    cap = N - 7
    # host-checked: the count is read back and nothing is written
    handle = ep.Handle.empty(w.num_ranks, w.num_tokens, w.num_channels, w.local_experts, cap, "cuda")
    recv_x = torch.zeros((cap, w.hidden), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ep.EpError) as e:
        ep.ep_dispatch(buf.ctx, inp.x_d, inp.topk_d, None, None, None, None, handle, recv_x, None,
                       None, cap, want_num_recv=True)
    assert e.value.status == 3
    assert not recv_x.any()
    # device-checked: rows below the capacity land, the rest are dropped and reported
    ep.ep_dispatch(buf.ctx, inp.x_d, inp.topk_d, None, None, None, None, handle, recv_x, None,
                   None, cap)
    assert buf.sync_status() == 3
    assert buf.sync_status() == 0          # the error word is cleared once read
    np.testing.assert_array_equal(u16(recv_x), o_recv_x[:cap])
    buf.destroy()


def test_bad_expert_id_is_reported(ep):
    w = W["tiny"]
    buf = make_buffer(ep, w)
    topk = torch.from_numpy(synth.topk_idx(w)).cuda()
    topk[1, 5, 0] = w.num_experts + 3
    buf.get_dispatch_layout(topk)
    assert buf.sync_status() == 4
    buf.destroy()


def test_misaligned_rows_are_rejected(ep):
    w = W["tiny"]
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    flat = torch.empty(inp.x_d.numel() + 8, dtype=torch.bfloat16, device="cuda")
    x_bad = flat[1:1 + inp.x_d.numel()].view(inp.x_d.shape)
    with pytest.raises(ep.EpError) as e:
        buf.dispatch(x_bad, inp.topk_d)
    assert e.value.status == 2
    buf.destroy()


def test_profile_counts_every_kernel(ep):
    w = W["tiny"]
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    ep.ep_profile_enable(buf.ctx, True)
    before = ep.kernel_launch_count()
    recv_x, _, recv_w, handle = buf.dispatch(inp.x_d, inp.topk_d, inp.weights_d)
    buf.combine(recv_x, handle, recv_w)
    buf.dispatch_cached(inp.x_d, handle)
    packed, _, llh = buf.low_latency_dispatch(inp.x_d, inp.topk_d)
    buf.low_latency_combine(packed, inp.topk_d, inp.weights_d, llh)
    buf.low_latency_dispatch(inp.x_d, inp.topk_d, use_fp8=True)
    mapping = torch.tensor([1, -1, 1, 3], dtype=torch.int32, device="cuda")
    ew = torch.ones((w.num_experts, 64), dtype=torch.bfloat16, device="cuda")
    red = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    buf.lb_prefetch_weights(red, ew, mapping)
    buf.lb_reduce_grads(red, ew, mapping)
    prof = ep.ep_profile_read(buf.ctx)
    assert ep.kernel_launch_count() - before == 12
    for kind in ep.PROFILE_KINDS:
        n, ms = prof[kind]
        assert n == (2 if kind == "ll_count" else 1) and ms > 0, kind
    buf.destroy()


FP8_CASES = [w for w in LL_CASES if w.hidden % 128 == 0]


@pytest.mark.parametrize("w", FP8_CASES, ids=ids(FP8_CASES))
def test_low_latency_fp8(ep, w):
    """FP8 packing: same slots as the bf16 form; codes and scales bit-exact."""
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    (codes, scales), count, (src_info, layout_range) = buf.low_latency_dispatch(
        inp.x_d, inp.topk_d, use_fp8=True)
    assert buf.sync_status() == 0
    ll = oracle.ll_dispatch(inp.x_u16, inp.topk, w.num_experts, w.tmax)
    np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
    np.testing.assert_array_equal(layout_range.cpu().numpy(), ll["layout_range"])
    c, sc, si = codes.cpu().numpy(), scales.cpu().numpy(), src_info.cpu().numpy()
    for d in range(w.num_ranks):
        for j in range(w.local_experts):
            n = int(ll["packed_recv_count"][d, j])
            if n == 0:
                continue
            np.testing.assert_array_equal(si[d, j, :n], ll["src_info"][d, j, :n])
            e_codes, e_scales = oracle.quantize_e4m3_blocks(ll["packed_recv_x"][d, j, :n], 128)
            np.testing.assert_array_equal(c[d, j, :n], e_codes, err_msg=f"codes of expert ({d},{j})")
            np.testing.assert_array_equal(sc[d, j, :n], e_scales, err_msg=f"scales of expert ({d},{j})")
    buf.destroy()


def test_low_latency_fp8_special_blocks(ep):
    """FP8 packing of the blocks a block quantiser can get wrong -- all +0 / -0,
    signed zeros around one +-1, a negative amax, N(0,1) x 2^124 and x 2^-100,
    E4M3 rounding ties, bf16 subnormals -- codes and scales bit-exact.  Rows of
    13 blocks: the last 512-channel step of a row is a quarter full."""
    w = W["ll"].scaled(num_tokens=24, hidden=13 * 128)
    inp = Inputs(w)
    x_u16 = synth.fp8_block_rows(w.seed + 11, w.num_ranks * w.num_tokens, w.hidden)
    x_d = to_bf16_tensor(x_u16.reshape(w.num_ranks, w.num_tokens, w.hidden)).cuda()
    buf = make_buffer(ep, w)
    (codes, scales), count, (src_info, _) = buf.low_latency_dispatch(x_d, inp.topk_d, use_fp8=True)
    assert buf.sync_status() == 0
    ll = oracle.ll_dispatch(x_u16.reshape(w.num_ranks, w.num_tokens, w.hidden), inp.topk,
                            w.num_experts, w.tmax)
    np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
    c, sc = codes.cpu().numpy(), scales.cpu().numpy()
    checked = 0
    for d in range(w.num_ranks):
        for j in range(w.local_experts):
            n = int(ll["packed_recv_count"][d, j])
            if n == 0:
                continue
            e_codes, e_scales = oracle.quantize_e4m3_blocks(ll["packed_recv_x"][d, j, :n], 128)
            np.testing.assert_array_equal(c[d, j, :n], e_codes, err_msg=f"codes of expert ({d},{j})")
            np.testing.assert_array_equal(sc[d, j, :n].view(np.uint32), e_scales.view(np.uint32),
                                          err_msg=f"scales of expert ({d},{j})")
            checked += n
    assert checked > 0
    buf.destroy()


def test_low_latency_fp8_rejects_unaligned_hidden(ep):
    w = next(c for c in LL_CASES if c.name == "ll-odd")      # hidden 40: not a multiple of 128
    assert w.hidden % 128 != 0
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    with pytest.raises(ep.EpError) as e:
        buf.low_latency_dispatch(inp.x_d, inp.topk_d, use_fp8=True)
    assert e.value.status == 1
    buf.destroy()


def test_low_latency_fp8_rejects_x_off_32_bytes(ep):
    """The FP8 copy reads x in 32-byte vectors: an x 16 bytes past a 32-byte boundary
    is refused before any launch (EP_ERR_ALIGNMENT); the bf16 form takes it."""
    w = W["ll"].scaled(num_tokens=8, hidden=256)
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    n = inp.x_d.numel()
    base = torch.empty(n + 16, dtype=torch.bfloat16, device="cuda")
    off = 8 if base.data_ptr() % 32 == 0 else 0          # elements: 16 bytes
    x = base[off:off + n].view(inp.x_d.shape)
    assert x.data_ptr() % 32 == 16
    x.copy_(inp.x_d)
    with pytest.raises(ep.EpError) as e:
        buf.low_latency_dispatch(x, inp.topk_d, use_fp8=True)
    assert e.value.status == 2
    packed, count, _ = buf.low_latency_dispatch(x, inp.topk_d)
    assert buf.sync_status() == 0
    ll = oracle.ll_dispatch(inp.x_u16, inp.topk, w.num_experts, w.tmax)
    np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
    buf.destroy()


@pytest.mark.parametrize("masked", [[3], [0, 15]], ids=["mask-3", "mask-0-15"])
def test_low_latency_rank_mask(ep, masked):
    """A rank marked failed on the host leaves the low-latency exchange; the other ranks'
    results equal the oracle's with that rank masked; unmask / clean restores it."""
    w = W["ll"].scaled(num_tokens=40, hidden=1024)
    R, E = w.num_ranks, w.num_experts
    inp = Inputs(w)
    buf = make_buffer(ep, w)
    for r in masked:
        buf.low_latency_update_mask_buffer(r, True)
    mask = buf.low_latency_query_mask_buffer().numpy()
    assert mask.tolist() == [int(r in masked) for r in range(R)]

    packed, count, (src_info, layout_range) = buf.low_latency_dispatch(inp.x_d, inp.topk_d)
    assert buf.sync_status() == 0
    ll = oracle.ll_dispatch(inp.x_u16, inp.topk, E, w.tmax, rank_mask=mask)
    np.testing.assert_array_equal(count.cpu().numpy(), ll["packed_recv_count"])
    np.testing.assert_array_equal(layout_range.cpu().numpy(), ll["layout_range"])
    p, si = u16(packed), src_info.cpu().numpy()
    for d in range(R):
        for j in range(w.local_experts):
            n = int(ll["packed_recv_count"][d, j])
            np.testing.assert_array_equal(si[d, j, :n], ll["src_info"][d, j, :n])
            np.testing.assert_array_equal(p[d, j, :n], ll["packed_recv_x"][d, j, :n])
    y_u16 = u16(synth.expert_rows(w.seed + 3, p.reshape(-1, w.hidden).shape[0], w.hidden)).reshape(p.shape)
    out = buf.low_latency_combine(to_bf16_tensor(y_u16).cuda(), inp.topk_d, inp.weights_d,
                                  (src_info, layout_range))
    args = (ll["src_info"], ll["layout_range"], E, w.tmax)
    got = u16(out)
    check_combine(f"ll combine, ranks {masked} masked", got,
                  oracle.ll_combine(y_u16, inp.topk, inp.weights, *args, rank_mask=mask, fp32=True),
                  oracle.ll_combine(y_u16, inp.topk, inp.weights, *args, rank_mask=mask),
                  oracle.ll_combine(bf16_abs(y_u16), inp.topk, np.abs(inp.weights), *args, rank_mask=mask),
                  w.topk)
    assert (got[mask.astype(bool)] == 0).all()

    (codes, scales), count8, _ = buf.low_latency_dispatch(inp.x_d, inp.topk_d, use_fp8=True)
    np.testing.assert_array_equal(count8.cpu().numpy(), ll["packed_recv_count"])
    c = codes.cpu().numpy()
    for d in range(R):
        for j in range(w.local_experts):
            n = int(ll["packed_recv_count"][d, j])
            if n:
                e_codes, _ = oracle.quantize_e4m3_blocks(ll["packed_recv_x"][d, j, :n], 128)
                np.testing.assert_array_equal(c[d, j, :n], e_codes)

    # recovery: unmask one rank, then clean all
    buf.low_latency_update_mask_buffer(masked[0], False)
    assert buf.low_latency_query_mask_buffer().numpy()[masked[0]] == 0
    buf.low_latency_clean_mask_buffer()
    assert not buf.low_latency_query_mask_buffer().numpy().any()
    _, count2, _ = buf.low_latency_dispatch(inp.x_d, inp.topk_d)
    np.testing.assert_array_equal(count2.cpu().numpy(),
                                  oracle.ll_dispatch(None, inp.topk, E, w.tmax, with_rows=False)["packed_recv_count"])
    assert buf.sync_status() == 0
    buf.destroy()


def test_low_latency_mask_rejects_bad_rank(ep):
    w = W["tiny"]
    buf = make_buffer(ep, w)
    with pytest.raises(ep.EpError):
        buf.low_latency_update_mask_buffer(w.num_ranks, True)
    buf.destroy()


@pytest.mark.parametrize("E,W,N", [(32, 7168 * 8, 12), (8, 24, 5), (4, 4096, 9)])
def test_load_balance_prefetch_and_reduce(ep, E, W, N):
    w = synth.Workload("lb", 4, E, 16, 64, 2, "uniform", 90)
    buf = make_buffer(ep, w)
    mapping = synth.redundancy_mapping(E, N, seed=E * 1000 + N, unused_prob=0.2)
    mapping[0] = mapping[1] = 2                    # an expert with several replicas
    ew = synth.expert_rows(91, E, W)
    before = synth.expert_rows(92, N, W)
    red = before.clone().cuda()
    buf.lb_prefetch_weights(red, ew.cuda(), torch.from_numpy(mapping).cuda())
    assert buf.sync_status() == 0
    np.testing.assert_array_equal(u16(red), oracle.lb_prefetch_weights(u16(ew), mapping, u16(before)))

    n_terms = 1 + int(np.bincount(mapping[mapping >= 0], minlength=E).max())
    untouched = np.setdiff1d(np.arange(E), mapping)
    for what, grads, rg in (("N(0,1) rows", u16(synth.expert_rows(93, E, W)), u16(synth.expert_rows(94, N, W))),
                            ("cancelling rows", synth.cancel_rows(95, E, W), synth.cancel_rows(96, N, W))):
        g_d = to_bf16_tensor(grads).cuda()
        buf.lb_reduce_grads(to_bf16_tensor(rg).cuda(), g_d, torch.from_numpy(mapping).cuda())
        assert buf.sync_status() == 0
        got = u16(g_d)
        check_combine(f"lb reduce E{E} W{W} N{N}, {what}", got,
                      oracle.lb_reduce_grads(rg, mapping, grads, fp32=True),
                      oracle.lb_reduce_grads(rg, mapping, grads),
                      oracle.lb_reduce_grads(bf16_abs(rg), mapping, bf16_abs(grads)), n_terms,
                      cancelling=what.startswith("cancelling"))
        np.testing.assert_array_equal(got[untouched], grads[untouched])
    buf.destroy()


def test_load_balance_bad_mapping_is_reported(ep):
    w = synth.Workload("lb", 4, 8, 16, 64, 2, "uniform", 90)
    buf = make_buffer(ep, w)
    ew = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    red = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    buf.lb_prefetch_weights(red, ew, torch.tensor([1, 8], dtype=torch.int32, device="cuda"))
    assert buf.sync_status() == 4
    with pytest.raises(ep.EpError) as e:               # 60 values per expert: not whole 16-byte vectors
        buf.lb_prefetch_weights(torch.zeros((2, 60), dtype=torch.bfloat16, device="cuda"),
                                torch.zeros((8, 60), dtype=torch.bfloat16, device="cuda"),
                                torch.tensor([1, 2], dtype=torch.int32, device="cuda"))
    assert e.value.status == 2
    buf.destroy()
