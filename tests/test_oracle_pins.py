"""Pins for the CPU oracle, checked against things other than the oracle itself.

* a hand-worked fixture (tests/golden/tiny_handle.txt);
* a second, independent formulation by brute force: one global stable sort of
  (destination, source, token) triples, pure Python, tiny inputs;
* closed forms: identity experts make the combine return fan-out * x, the
  low-latency combine with weights 1/8 returns (valid slots / 8) * x;
* exact integer-valued rows, so any dropped, doubled or misplaced term shows;
* invariants (counts, monotone prefixes, permutation inverses);
* special cases: one rank, top-1, all slots masked, no tokens, more channels
  than tokens;
* the bf16 rounding step against exact rational arithmetic and against torch.

All CPU, no GPU.
"""
import bisect
import fractions
import itertools
import os
import struct

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import load_golden_fp32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_handle.txt")


# ----------------------------------------------------------------------------
# helpers written for the tests (independent of the oracle)

def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_torch(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits via torch's conversion (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def brute_handle(topk, E, C):
    """Independent formulation: sort all (d, s, t) triples once."""
    R, T, K = topk.shape
    L = E // R
    triples = []
    for s in range(R):
        for t in range(T):
            dests = sorted({int(e) // L for e in topk[s, t] if e != -1})
            for d in dests:
                triples.append((d, s, t))
    triples.sort()
    N = [0] * R
    for d, _, _ in triples:
        N[d] += 1
    off = [0]
    for d in range(R):
        off.append(off[-1] + N[d])
    send_head = -np.ones((R, T, R), np.int64)
    recv_src = np.zeros(len(triples), np.int64)
    for row, (d, s, t) in enumerate(triples):
        send_head[s, t, d] = row - off[d]
        recv_src[row] = t
    q = -(-T // C) if T else 0
    start = [min(c * q, T) for c in range(C + 1)]
    # recv_channel_prefix[d][s][c] = number of triples that sort before (d, s, start(c))
    rcp = np.zeros((R, R, C), np.int64)
    cp = np.zeros((R, R, C), np.int64)
    for d in range(R):
        for s in range(R):
            for c in range(C):
                rcp[d, s, c] = bisect.bisect_left(triples, (d, s, start[c])) - off[d]
                cp[s, d, c] = sum(1 for (dd, ss, tt) in triples
                                  if dd == d and ss == s and tt < start[c + 1])
    rp = np.zeros((R, R), np.int64)
    for i in range(R):
        for d in range(R):
            rp[i, d] = sum(1 for (dd, ss, _) in triples if dd == d and ss <= i)
    return dict(send_head=send_head, recv_src_idx=recv_src, recv_rank_offset=np.array(off),
                rank_prefix_matrix=rp, channel_prefix_matrix=cp,
                recv_channel_prefix_matrix=rcp, triples=triples)


def brute_ll(topk, E):
    R, T, K = topk.shape
    L = E // R
    lists = {e: [] for e in range(E)}
    for s in range(R):
        for t in range(T):
            for e in set(int(v) for v in topk[s, t] if v != -1):
                lists[e].append((s, t))
    for e in lists:
        lists[e].sort()
    return lists


def random_topk(rng, R, E, T, K, mask_p=0.0, distinct=True):
    out = np.empty((R, T, K), np.int64)
    for s in range(R):
        for t in range(T):
            if distinct:
                out[s, t] = rng.choice(E, size=K, replace=False)
            else:
                out[s, t] = rng.integers(0, E, size=K)
    if mask_p:
        out[rng.random(out.shape) < mask_p] = -1
    return out


def run_oracle_dispatch(topk, E, C, x=None, w=None):
    ntr, nte, tin = oracle.layout(topk, E)
    h = oracle.dispatch_handle(tin, nte, C)
    rows = None
    if x is not None:
        rows = oracle.dispatch_rows(x, topk, w, h, E)
    return ntr, nte, tin, h, rows


# ----------------------------------------------------------------------------
# hand-worked fixture

def load_golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [int(v) for v in rest]
    return vals


def test_golden_layout_and_handle():
    g = load_golden()
    R, E, T, K, C = g["R"][0], g["E"][0], g["T"][0], g["K"][0], g["C"][0]
    topk = np.array(g["topk_idx"], np.int64).reshape(R, T, K)
    ntr, nte, tin = oracle.layout(topk, E)
    assert tin.ravel().tolist() == g["is_token_in_rank"]
    assert ntr.ravel().tolist() == g["num_tokens_per_rank"]
    assert nte.ravel().tolist() == g["num_tokens_per_expert"]
    h = oracle.dispatch_handle(tin, nte, C)
    for key in ("send_head", "recv_rank_offset", "recv_src_idx", "rank_prefix_matrix",
                "channel_prefix_matrix", "recv_channel_prefix_matrix",
                "num_recv_tokens_per_expert"):
        assert h[key].ravel().tolist() == g[key], key


def test_golden_rows_and_combine():
    g = load_golden()
    R, E, T, K, C, H = (g[k][0] for k in ("R", "E", "T", "K", "C", "H"))
    topk = np.array(g["topk_idx"], np.int64).reshape(R, T, K)
    xv = np.array(g["x"], np.float32).reshape(R, T, H)
    x = f32_to_bf16_torch(xv)
    w = np.full((R, T, K), 0.5, np.float32)
    _, _, _, h, (recv_x, recv_idx, recv_w) = run_oracle_dispatch(topk, E, C, x, w)
    assert recv_idx.ravel().tolist() == g["recv_topk_idx"]
    out, _ = oracle.combine(recv_x, h)
    assert bf16_to_f64(out).ravel().tolist() == g["combine_identity"]


def test_golden_ll():
    g = load_golden()
    R, E, T, K, H, Tmax = (g[k][0] for k in ("R", "E", "T", "K", "H", "TMAX"))
    topk = np.array(g["topk_idx"], np.int64).reshape(R, T, K)
    x = f32_to_bf16_torch(np.array(g["x"], np.float32).reshape(R, T, H))
    ll = oracle.ll_dispatch(x, topk, E, Tmax)
    assert ll["packed_recv_count"].ravel().tolist() == g["ll_count"]
    L = E // R
    for e in range(E):
        n = g["ll_count"][e]
        assert ll["src_info"][e // L, e % L, :n].tolist() == g[f"ll_src_info_e{e}"]
    assert ll["layout_range"].ravel().tolist() == g["ll_layout_range"]


# ----------------------------------------------------------------------------
# brute force (independent sort-based formulation)

@pytest.mark.parametrize("R,E,T,K,C,mask_p", [
    (2, 8, 13, 2, 3, 0.0), (4, 16, 9, 3, 2, 0.1), (3, 9, 7, 4, 5, 0.3),
    (1, 4, 6, 2, 2, 0.2), (5, 10, 4, 2, 7, 0.0), (8, 32, 11, 8, 3, 0.05),
])
def test_handle_matches_sort_formulation(R, E, T, K, C, mask_p):
    rng = np.random.default_rng(R * 1000 + E * 10 + T)
    topk = random_topk(rng, R, E, T, K, mask_p)
    ntr, nte, tin, h, _ = run_oracle_dispatch(topk, E, C)
    b = brute_handle(topk, E, C)
    for key in ("send_head", "recv_src_idx", "recv_rank_offset", "rank_prefix_matrix",
                "channel_prefix_matrix", "recv_channel_prefix_matrix"):
        np.testing.assert_array_equal(h[key], b[key], err_msg=key)
    # layout by brute counting
    L = E // R
    for s in range(R):
        for t in range(T):
            dests = {int(e) // L for e in topk[s, t] if e != -1}
            assert [int(v) for v in tin[s, t]] == [int(d in dests) for d in range(R)]
    exp_nte = np.zeros((R, E), np.int64)
    for s, t, k in itertools.product(range(R), range(T), range(K)):
        if topk[s, t, k] != -1:
            exp_nte[s, topk[s, t, k]] += 1
    np.testing.assert_array_equal(nte, exp_nte)
    np.testing.assert_array_equal(h["num_recv_tokens_per_expert"],
                                  exp_nte.sum(0).reshape(R, L))


def _random_shape(seed):
    rng = np.random.default_rng(0xC0FFEE + seed)
    R = int(rng.integers(1, 9))
    E = R * int(rng.integers(1, 5))
    T = int(rng.integers(0, 21))
    K = int(rng.integers(1, min(E, 6) + 1))
    C = int(rng.integers(1, 9))
    mask_p = float(rng.choice([0.0, 0.2, 0.5, 1.0]))
    distinct = bool(rng.integers(0, 2))
    return rng, R, E, T, K, C, mask_p, distinct


@pytest.mark.parametrize("seed", range(40))
def test_random_shapes_match_the_independent_formulations(seed):
    """Forty seeded tiny shapes, T = 0, fully masked and repeated experts included:
    the handle against the sort formulation, the low-latency lists against the
    per-expert enumeration."""
    rng, R, E, T, K, C, mask_p, distinct = _random_shape(seed)
    topk = random_topk(rng, R, E, T, K, mask_p, distinct=distinct)
    if distinct:
        _, _, _, h, _ = run_oracle_dispatch(topk, E, C)
        b = brute_handle(topk, E, C)
        for key in ("send_head", "recv_src_idx", "recv_rank_offset", "rank_prefix_matrix",
                    "channel_prefix_matrix", "recv_channel_prefix_matrix"):
            np.testing.assert_array_equal(h[key], b[key], err_msg=f"{key} {(R, E, T, K, C, mask_p)}")
    x = f32_to_bf16_torch(rng.standard_normal((R, T, 8)).astype(np.float32))
    ll = oracle.ll_dispatch(x, topk, E, max(T, 1))
    L = E // R
    for e, lst in brute_ll(topk, E).items():
        d, j = divmod(e, L)
        assert ll["packed_recv_count"][d, j] == len(lst)
        for slot, (s_, t) in enumerate(lst):
            assert ll["src_info"][d, j, slot] == t
        for s_ in range(R):
            begin = sum(1 for (ss, _) in lst if ss < s_)
            cnt = sum(1 for (ss, _) in lst if ss == s_)
            assert ll["layout_range"][d, j, s_].tolist() == [begin, cnt]


def test_dispatch_rows_and_combine_integer_rows():
    """Rows carry exact small integers; the combine sum and every row copy are exact."""
    rng = np.random.default_rng(7)
    R, E, T, K, C, H = 4, 16, 10, 3, 3, 16
    topk = random_topk(rng, R, E, T, K, mask_p=0.15)
    w = rng.random((R, T, K)).astype(np.float32)
    xv = rng.integers(-20, 21, size=(R, T, H)).astype(np.float32)
    x = f32_to_bf16_torch(xv)
    _, _, tin, h, (recv_x, recv_idx, recv_w) = run_oracle_dispatch(topk, E, C, x, w)
    b = brute_handle(topk, E, C)
    L = E // R
    for row, (d, s, t) in enumerate(b["triples"]):
        np.testing.assert_array_equal(recv_x[row], x[s, t])
        for k in range(K):
            e = topk[s, t, k]
            here = e != -1 and e // L == d
            assert recv_idx[row, k] == (e % L if here else -1)
            assert recv_w[row, k] == (w[s, t, k] if here else 0.0)
    # Each received row gets its own integer signature; the combine must add
    # exactly the rows that belong to the token.
    yv = rng.integers(-8, 9, size=recv_x.shape).astype(np.float32)
    y = f32_to_bf16_torch(yv)
    out, out_w = oracle.combine(y, h, recv_w)
    exp = np.zeros((R, T, H))
    for row, (d, s, t) in enumerate(b["triples"]):
        exp[s, t] += yv[row]
    np.testing.assert_array_equal(bf16_to_f64(out), exp)
    # weights: exactly one destination owns each valid slot
    exp_w = np.where(topk != -1, w, 0.0).astype(np.float32)
    np.testing.assert_array_equal(out_w, exp_w)


def test_combine_identity_experts_closed_form():
    """y = recv_x  =>  out = bf16(fan-out * x) (exact: fan-out * x fits in fp32)."""
    w_ = synth.WORKLOADS["dsv3"].scaled(num_tokens=40, hidden=64)
    topk = synth.topk_idx(w_)
    x = synth.hidden_rows(w_).view(torch.int16).numpy().view(np.uint16).copy()
    x[0, :5, :3] = 0x8000          # negative zeros: a sum that starts at +0 stays +0
    x[1, :5, :3] = 0x0000
    _, _, tin, h, (recv_x, _, _) = run_oracle_dispatch(topk, w_.num_experts, w_.num_channels, x)
    out, _ = oracle.combine(recv_x, h)
    fan = tin.sum(-1).astype(np.float32)
    exp = f32_to_bf16_torch(fan[..., None] * bf16_to_f64(x).astype(np.float32))
    exp[exp == 0x8000] = 0
    np.testing.assert_array_equal(out, exp)
    assert (out[0, :5, :3] == 0).all()


def test_combine_bias_closed_form():
    rng = np.random.default_rng(3)
    R, E, T, K, C, H = 2, 4, 5, 2, 2, 8
    topk = random_topk(rng, R, E, T, K)
    b0v = rng.integers(-5, 6, (R, T, H)).astype(np.float32)
    b1v = rng.integers(-5, 6, (R, T, H)).astype(np.float32)
    x = f32_to_bf16_torch(np.zeros((R, T, H), np.float32))
    _, _, _, h, (recv_x, _, _) = run_oracle_dispatch(topk, E, C, x)
    out, _ = oracle.combine(recv_x, h, bias0=f32_to_bf16_torch(b0v), bias1=f32_to_bf16_torch(b1v))
    np.testing.assert_array_equal(bf16_to_f64(out), b0v + b1v)


def test_combine_token_subset_matches_full():
    w_ = synth.WORKLOADS["tiny"]
    topk = synth.topk_idx(w_)
    x = synth.hidden_rows(w_).view(torch.int16).numpy().view(np.uint16)
    _, _, _, h, (recv_x, _, recv_w) = run_oracle_dispatch(
        topk, w_.num_experts, w_.num_channels, x, synth.topk_weights(w_))
    full, full_w = oracle.combine(recv_x, h, recv_w)
    toks = np.array([5, 0, 127, 64, 3])
    part, part_w = oracle.combine(recv_x, h, recv_w, tokens=toks)
    np.testing.assert_array_equal(part, full.reshape(-1, w_.hidden)[toks])
    np.testing.assert_array_equal(part_w, full_w.reshape(-1, w_.topk)[toks])


# ----------------------------------------------------------------------------
# invariants on the synthetic workloads (small token counts)

@pytest.mark.parametrize("name", ["tiny", "dsv3", "ll", "zipf", "reuse"])
def test_layout_and_handle_invariants(name):
    w_ = synth.WORKLOADS[name]
    w_ = w_.scaled(num_tokens=min(w_.num_tokens, 300), hidden=8)
    topk = synth.topk_idx(w_)
    R, T, K = topk.shape
    ntr, nte, tin, h, _ = run_oracle_dispatch(topk, w_.num_experts, w_.num_channels)
    L = w_.local_experts
    valid = topk != -1
    np.testing.assert_array_equal(ntr.sum(1), tin.reshape(R, -1).sum(1))
    np.testing.assert_array_equal(nte.sum(1), valid.reshape(R, -1).sum(1))
    assert (ntr <= nte.reshape(R, R, L).sum(-1)).all()
    rp, cp, rcp = h["rank_prefix_matrix"], h["channel_prefix_matrix"], h["recv_channel_prefix_matrix"]
    N = h["recv_rank_offset"][1:] - h["recv_rank_offset"][:-1]
    assert (np.diff(rp, axis=0) >= 0).all()
    np.testing.assert_array_equal(rp[-1], N)
    np.testing.assert_array_equal(rp[-1], ntr.sum(0))
    assert (np.diff(cp, axis=2) >= 0).all()
    np.testing.assert_array_equal(cp[:, :, -1], ntr)
    assert (np.diff(rcp.reshape(R, -1), axis=1) >= 0).all()
    # permutation inverse: recv_src_idx o send_head = token id, rows form a bijection
    sh = h["send_head"]
    seen = np.zeros(int(h["recv_rank_offset"][-1]), bool)
    for d in range(R):
        s_idx, t_idx = np.nonzero(sh[:, :, d] >= 0)
        rows = h["recv_rank_offset"][d] + sh[s_idx, t_idx, d]
        np.testing.assert_array_equal(h["recv_src_idx"][rows], t_idx)
        assert not seen[rows].any()
        seen[rows] = True
        np.testing.assert_array_equal(sh[:, :, d] >= 0, tin[:, :, d].astype(bool))
    assert seen.all()
    # the first token of each non-empty (source, channel) block sits at recv_channel_prefix
    C = w_.num_channels
    q = -(-T // C)
    for d in range(R):
        for s in range(R):
            for c in range(C):
                lo, hi = min(c * q, T), min((c + 1) * q, T)
                members = np.nonzero(tin[s, lo:hi, d])[0]
                if members.size:
                    assert sh[s, lo + members[0], d] == rcp[d, s, c]


# ----------------------------------------------------------------------------
# special cases

def test_single_rank_is_identity_on_routed_tokens():
    rng = np.random.default_rng(11)
    topk = random_topk(rng, 1, 6, 20, 2, mask_p=0.4)
    x = f32_to_bf16_torch(rng.standard_normal((1, 20, 8)).astype(np.float32))
    _, _, tin, h, (recv_x, _, _) = run_oracle_dispatch(topk, 6, 4, x)
    routed = np.nonzero(tin[0, :, 0])[0]
    np.testing.assert_array_equal(h["recv_src_idx"], routed)
    np.testing.assert_array_equal(recv_x, x[0, routed])


def test_top1_combine_of_identity_returns_x():
    rng = np.random.default_rng(12)
    R, E, T, H = 4, 8, 16, 32
    topk = random_topk(rng, R, E, T, 1, mask_p=0.2)
    x = f32_to_bf16_torch(rng.standard_normal((R, T, H)).astype(np.float32))
    _, _, tin, h, (recv_x, _, _) = run_oracle_dispatch(topk, E, 3, x)
    out, _ = oracle.combine(recv_x, h)
    routed = tin.any(-1)
    np.testing.assert_array_equal(out[routed], x[routed])
    assert (out[~routed] == 0).all()


def test_all_masked_and_empty():
    R, E, T, K, C, H = 3, 6, 5, 2, 4, 8
    topk = -np.ones((R, T, K), np.int64)
    x = np.ones((R, T, H), np.uint16) * 0x3f80
    ntr, nte, tin, h, (recv_x, _, _) = run_oracle_dispatch(topk, E, C, x)
    assert ntr.sum() == 0 and nte.sum() == 0 and tin.sum() == 0
    assert h["recv_rank_offset"].tolist() == [0] * (R + 1)
    assert (h["send_head"] == -1).all()
    assert not h["rank_prefix_matrix"].any() and not h["channel_prefix_matrix"].any()
    out, _ = oracle.combine(np.zeros((0, H), np.uint16), h)
    assert (out == 0).all()
    # no tokens at all
    topk0 = np.zeros((R, 0, K), np.int64)
    ntr, nte, tin, h, _ = run_oracle_dispatch(topk0, E, C)
    assert h["recv_rank_offset"].tolist() == [0] * (R + 1)
    assert not h["recv_channel_prefix_matrix"].any()


def test_more_channels_than_tokens():
    rng = np.random.default_rng(5)
    topk = random_topk(rng, 2, 4, 3, 2)
    _, _, _, h, _ = run_oracle_dispatch(topk, 4, 8)
    b = brute_handle(topk, 4, 8)
    np.testing.assert_array_equal(h["channel_prefix_matrix"], b["channel_prefix_matrix"])
    np.testing.assert_array_equal(h["recv_channel_prefix_matrix"], b["recv_channel_prefix_matrix"])


def test_bad_expert_id_is_rejected():
    topk = np.array([[[0, 9]]], np.int64)
    with pytest.raises(oracle.OracleError):
        oracle.layout(topk, 4)
    with pytest.raises(oracle.OracleError):
        oracle.layout(np.array([[[-2, 0]]], np.int64), 4)


# ----------------------------------------------------------------------------
# low-latency path

@pytest.mark.parametrize("R,E,T,K,Tmax,distinct", [
    (2, 8, 12, 2, 12, True), (4, 16, 9, 4, 11, True), (3, 6, 10, 3, 10, False),
])
def test_ll_dispatch_matches_lists(R, E, T, K, Tmax, distinct):
    rng = np.random.default_rng(R + E + T)
    topk = random_topk(rng, R, E, T, K, mask_p=0.1, distinct=distinct)
    H = 8
    x = f32_to_bf16_torch(rng.standard_normal((R, T, H)).astype(np.float32))
    ll = oracle.ll_dispatch(x, topk, E, Tmax)
    lists = brute_ll(topk, E)
    L = E // R
    total = 0
    for e, lst in lists.items():
        d, j = divmod(e, L)
        assert ll["packed_recv_count"][d, j] == len(lst)
        total += len(lst)
        for slot, (s, t) in enumerate(lst):
            assert ll["src_info"][d, j, slot] == t
            np.testing.assert_array_equal(ll["packed_recv_x"][d, j, slot], x[s, t])
        for s in range(R):
            begin = sum(1 for (ss, _) in lst if ss < s)
            cnt = sum(1 for (ss, _) in lst if ss == s)
            assert ll["layout_range"][d, j, s].tolist() == [begin, cnt]
    assert total == sum(len({int(v) for v in topk[s, t] if v != -1})
                        for s in range(R) for t in range(T))


def test_ll_combine_closed_form_uniform_weights():
    """Weights 1/8 on identity experts: out = bf16((valid slots / 8) * x), exactly."""
    w_ = synth.WORKLOADS["ll"].scaled(num_tokens=12, hidden=32)
    topk = synth.topk_idx(w_)
    rng = np.random.default_rng(1)
    topk[rng.random(topk.shape) < 0.2] = -1
    x = synth.hidden_rows(w_).view(torch.int16).numpy().view(np.uint16)
    ll = oracle.ll_dispatch(x, topk, w_.num_experts, w_.tmax)
    wts = np.full(topk.shape, 0.125, np.float32)
    out = oracle.ll_combine(ll["packed_recv_x"], topk, wts, ll["src_info"], ll["layout_range"],
                            w_.num_experts, w_.tmax)
    n_valid = (topk != -1).sum(-1).astype(np.float32)
    exp = f32_to_bf16_torch(n_valid[..., None] / 8 * bf16_to_f64(x).astype(np.float32))
    np.testing.assert_array_equal(out, exp)


def test_ll_combine_integer_rows_weighted():
    """Per-slot integer rows and power-of-two weights: every term is exact."""
    rng = np.random.default_rng(21)
    R, E, T, K, H = 3, 12, 7, 3, 4
    topk = random_topk(rng, R, E, T, K, mask_p=0.2)
    ll = oracle.ll_dispatch(None, topk, E, T, with_rows=False)
    L = E // R
    cap = R * T
    yv = rng.integers(-6, 7, size=(R, L, cap, H)).astype(np.float32)
    y = f32_to_bf16_torch(yv)
    wts = (2.0 ** rng.integers(-3, 2, size=topk.shape)).astype(np.float32)
    out = oracle.ll_combine(y, topk, wts, ll["src_info"], ll["layout_range"], E, T)
    lists = brute_ll(topk, E)
    exp = np.zeros((R, T, H))
    for s in range(R):
        for t in range(T):
            for k in range(K):
                e = int(topk[s, t, k])
                if e == -1:
                    continue
                slot = lists[e].index((s, t))
                exp[s, t] += float(wts[s, t, k]) * yv[e // L, e % L, slot]
    np.testing.assert_array_equal(bf16_to_f64(out), exp)


# ----------------------------------------------------------------------------
# bf16 rounding

def _exact_nearest_bf16(v: float) -> float:
    """Nearest bf16 by exact rational comparison of the two bracketing values."""
    if v == 0:
        return v
    f = fractions.Fraction(v)
    a = abs(f)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    q = fractions.Fraction(2) ** max(e - 7, -133)        # spacing of bf16 values here
    lo = (abs(f) // q) * q
    hi = lo + q
    dlo, dhi = abs(f) - lo, hi - abs(f)
    if dlo < dhi:
        r = lo
    elif dhi < dlo:
        r = hi
    else:
        r = lo if (lo / q) % 2 == 0 else hi
    r = float(r)
    return -r if v < 0 else r


def test_round_bf16_against_exact_and_torch():
    rng = np.random.default_rng(0)
    f32 = rng.standard_normal(20000).astype(np.float32)
    ties = (np.frombuffer(f32.tobytes(), np.uint32) & 0xFFFF0000 | 0x8000).view(np.float32)
    vals32 = np.concatenate([f32, ties, np.float32([1e-40, -3e-39, 3.0e38, 1.0, -0.0])])
    np.testing.assert_array_equal(oracle.round_bf16(vals32.astype(np.float64)),
                                  f32_to_bf16_torch(vals32))
    # doubles that are not float32 values: one-step rounding must beat double rounding
    dbl = np.concatenate([
        rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000),
        np.array([1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 2.0 ** -8 - 2.0 ** -40,
                  1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)]),
    ])
    got = bf16_to_f64(oracle.round_bf16(dbl))
    exp = np.array([_exact_nearest_bf16(float(v)) for v in dbl])
    np.testing.assert_array_equal(got, exp)
    assert struct.pack(">H", int(oracle.round_bf16(np.array([1.0 + 2.0 ** -8 + 2.0 ** -40]))[0])) \
        == b"\x3f\x81"


# ----------------------------------------------------------------------------
# FP8 (E4M3) block quantisation of the low-latency path

def _e4m3_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    return codes, vals


def test_e4m3_encoder_against_torch_and_ties():
    rng = np.random.default_rng(4)
    v32 = np.concatenate([rng.uniform(-448, 448, 50000), rng.standard_normal(50000) * 0.02]).astype(np.float32)
    np.testing.assert_array_equal(oracle.fp8_e4m3_encode(v32.astype(np.float64)),
                                  torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    codes, vals = _e4m3_values()
    finite = ~np.isnan(vals)
    np.testing.assert_array_equal(oracle.fp8_e4m3_encode(vals[finite]), codes[finite])
    # exact midpoints between neighbouring positive values round to the even code
    pos = np.sort(vals[finite & (vals > 0)])
    mids = (pos[:-1] + pos[1:]) / 2
    got = oracle.fp8_e4m3_encode(mids)
    lo = oracle.fp8_e4m3_encode(pos[:-1])
    hi = oracle.fp8_e4m3_encode(pos[1:])
    np.testing.assert_array_equal(got, np.where(lo % 2 == 0, lo, hi))
    # saturation at the largest finite value, both signs
    assert oracle.fp8_e4m3_encode(np.array([448.0, 463.9, 1e6, -1e6])).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]


def test_block_quantisation_closed_forms():
    H = 256
    # block 0: amax 56 -> scale 0.125 exactly; codes are e4m3(8 x) with 8 x exact in E4M3
    b0 = np.array([56.0, -56.0, 1.0, -0.5, 0.25, 3.0, 0.0, 7.0] * 16, np.float32)
    # block 1: all zero -> scale 1, codes 0
    b1 = np.zeros(128, np.float32)
    x = f32_to_bf16_torch(np.concatenate([b0, b1])[None, :])
    codes, scales = oracle.quantize_e4m3_blocks(x, 128)
    assert scales.tolist() == [[0.125, 1.0]]
    np.testing.assert_array_equal(codes[0, :128], oracle.fp8_e4m3_encode(8.0 * b0.astype(np.float64)))
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xFE          # amax maps to +-448
    assert not codes[0, 128:].any()


def test_block_quantisation_error_bound():
    rng = np.random.default_rng(9)
    x = f32_to_bf16_torch(rng.standard_normal((64, 512)).astype(np.float32))
    codes, scales = oracle.quantize_e4m3_blocks(x, 128)
    _, vals = _e4m3_values()
    deq = vals[codes] * np.repeat(scales.astype(np.float64), 128, axis=1)
    xf = bf16_to_f64(x)
    q = np.abs(xf) / np.repeat(scales.astype(np.float64), 128, axis=1)
    e = np.floor(np.log2(np.maximum(q, 2.0 ** -6)))
    half_step = 2.0 ** (e - 3) / 2 * np.repeat(scales.astype(np.float64), 128, axis=1)
    # half an E4M3 step, plus the fp32 roundings of 448/amax, amax/448 and the product
    assert (np.abs(deq - xf) <= half_step + 2.0 ** -21 * np.abs(xf) + 1e-30).all()
    # the largest element of each block is encoded as +-448
    blocks = np.abs(xf).reshape(64, 4, 128)
    arg = blocks.argmax(-1)
    c = codes.reshape(64, 4, 128)
    picked = np.take_along_axis(c, arg[..., None], -1)[..., 0]
    assert np.isin(picked, [0x7E, 0xFE]).all()


# ----------------------------------------------------------------------------
# dynamic rank masking (low-latency path)

@pytest.mark.parametrize("masked", [[1], [0, 3], [2, 3]])
def test_ll_rank_mask_equals_dropping_the_slots(masked):
    """Masking rank r is the same as dropping every slot that leaves from or goes to r;
    the tokens of a masked source rank combine to +0."""
    rng = np.random.default_rng(sum(masked) + 17)
    R, E, T, K, H = 4, 16, 9, 3, 8
    L = E // R
    topk = random_topk(rng, R, E, T, K, mask_p=0.1)
    x = f32_to_bf16_torch(rng.integers(-5, 6, (R, T, H)).astype(np.float32))
    wts = (2.0 ** rng.integers(-2, 2, topk.shape)).astype(np.float32)
    mask = np.zeros(R, np.int32)
    mask[masked] = 1
    dropped = topk.copy()
    for s in range(R):
        for t in range(T):
            for k in range(K):
                e = dropped[s, t, k]
                if e != -1 and (mask[s] or mask[e // L]):
                    dropped[s, t, k] = -1
    a = oracle.ll_dispatch(x, topk, E, T, rank_mask=mask)
    b = oracle.ll_dispatch(x, dropped, E, T)
    for key in ("packed_recv_count", "layout_range", "src_info", "packed_recv_x"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)
    yv = rng.integers(-4, 5, a["packed_recv_x"].shape).astype(np.float32)
    y = f32_to_bf16_torch(yv)
    out_a = oracle.ll_combine(y, topk, wts, a["src_info"], a["layout_range"], E, T, rank_mask=mask)
    out_b = oracle.ll_combine(y, dropped, wts, b["src_info"], b["layout_range"], E, T)
    np.testing.assert_array_equal(out_a, out_b)
    assert (out_a[mask.astype(bool)] == 0).all()
    # no expert on a masked rank receives anything
    assert (a["packed_recv_count"][mask.astype(bool)] == 0).all()


# ----------------------------------------------------------------------------
# load balance: redundant-expert weight prefetch and gradient reduction

def test_lb_prefetch_is_a_gather():
    rng = np.random.default_rng(31)
    E, W, N = 6, 40, 9
    ew = rng.integers(0, 1 << 16, (E, W)).astype(np.uint16)
    mapping = rng.integers(-1, E, N).astype(np.int32)
    before = rng.integers(0, 1 << 16, (N, W)).astype(np.uint16)
    out = oracle.lb_prefetch_weights(ew, mapping, before)
    for i in range(N):
        np.testing.assert_array_equal(out[i], ew[mapping[i]] if mapping[i] >= 0 else before[i])


def test_lb_reduce_integer_rows_exact():
    rng = np.random.default_rng(32)
    E, W, N = 5, 24, 11
    mapping = rng.integers(-1, E, N).astype(np.int32)
    g = rng.integers(-20, 21, (E, W)).astype(np.float32)
    r = rng.integers(-20, 21, (N, W)).astype(np.float32)
    out = oracle.lb_reduce_grads(f32_to_bf16_torch(r), mapping, f32_to_bf16_torch(g))
    exp = g.astype(np.float64).copy()
    for i in range(N):
        if mapping[i] >= 0:
            exp[mapping[i]] += r[i]
    np.testing.assert_array_equal(bf16_to_f64(out), exp)
    untouched = [e for e in range(E) if e not in set(mapping.tolist())]
    for e in untouched:
        np.testing.assert_array_equal(out[e], f32_to_bf16_torch(g[e]))


def test_lb_reduce_rounds_once():
    # 1 + 3 * 2^-8 is a tie between 1 + 2^-7 and 1 + 2^-6 and rounds to the even one, 1 + 2^-6;
    # rounding after every addition would give 1 (each 1 + 2^-8 ties back down to 1)
    g = f32_to_bf16_torch(np.array([[1.0]], np.float32))
    r = f32_to_bf16_torch(np.full((3, 1), 2.0 ** -8, np.float32))
    out = oracle.lb_reduce_grads(r, np.zeros(3, np.int32), g)
    assert bf16_to_f64(out)[0, 0] == 1.0 + 2.0 ** -6
    with pytest.raises(oracle.OracleError):
        oracle.lb_reduce_grads(r, np.array([0, 9, 0], np.int32), g)


# ----------------------------------------------------------------------------
# fixed-order fp32 reductions (the arithmetic the method performs)

def _f32(bits):
    return np.array(bits, np.uint32).view(np.float32)


def test_golden_fp32_combine_order():
    """Ascending destination ranks, then bias0, then bias1, in binary32 from +0:
    the hand-worked cancellation cases of tests/golden/fp32_order.txt."""
    g = load_golden_fp32()
    R, T, H, K = (g[f"combine_{k}"][0] for k in ("R", "T", "H", "K"))
    h = {"send_head": np.array(g["combine_send_head"], np.int32).reshape(R, T, R),
         "recv_rank_offset": np.array(g["combine_recv_rank_offset"], np.int64)}
    y = np.array(g["combine_y"], np.uint16).reshape(-1, H)
    b0 = np.array(g["combine_bias0"], np.uint16).reshape(R, T, H)
    b1 = np.array(g["combine_bias1"], np.uint16).reshape(R, T, H)
    rw = _f32(g["combine_recv_w"]).reshape(-1, K)
    out, out_w = oracle.combine(y, h, rw, bias0=b0, bias1=b1, fp32=True)
    assert out.ravel().tolist() == g["combine_out_fp32"]
    assert out_w.ravel().view(np.uint32).tolist() == g["combine_w_fp32"]
    out, out_w = oracle.combine(y, h, rw, bias0=b0, bias1=b1)
    assert out.ravel().tolist() == g["combine_out_exact"]
    assert out_w.ravel().view(np.uint32).tolist() == g["combine_w_exact"]


def test_golden_fp32_ll_combine_order_and_fma():
    """Ascending expert id (not k), one fused multiply-add per slot."""
    g = load_golden_fp32()
    R, E, T, K, Tmax, H = (g[f"ll_{k}"][0] for k in ("R", "E", "T", "K", "TMAX", "H"))
    topk = np.array(g["ll_topk_idx"], np.int64).reshape(R, T, K)
    ll = oracle.ll_dispatch(None, topk, E, Tmax, with_rows=False)
    y = np.array(g["ll_y"], np.uint16).reshape(R, E // R, R * Tmax, H)
    w = _f32(g["ll_w"]).reshape(R, T, K)
    out = oracle.ll_combine(y, topk, w, ll["src_info"], ll["layout_range"], E, Tmax, fp32=True)
    assert out.ravel().tolist() == g["ll_out_fp32"]
    out = oracle.ll_combine(y, topk, w, ll["src_info"], ll["layout_range"], E, Tmax)
    assert out.ravel().tolist() == g["ll_out_exact"]


def test_golden_fp32_lb_reduce_order():
    g = load_golden_fp32()
    m = np.array(g["lb_mapping"], np.int32)
    grads = np.array(g["lb_grads"], np.uint16).reshape(1, 1)
    red = np.array(g["lb_redundant"], np.uint16).reshape(-1, 1)
    assert oracle.lb_reduce_grads(red, m, grads, fp32=True).ravel().tolist() == g["lb_out_fp32"]
    assert oracle.lb_reduce_grads(red, m, grads).ravel().tolist() == g["lb_out_exact"]


def test_fp32_reductions_exact_on_integer_rows():
    """Small integers and power-of-two weights: every binary32 operation is exact, so
    the fixed-order results equal the exact sums counted by brute force."""
    rng = np.random.default_rng(41)
    R, E, T, K, C, H = 4, 16, 10, 3, 3, 16
    topk = random_topk(rng, R, E, T, K, mask_p=0.15)
    w = (2.0 ** rng.integers(-4, 3, (R, T, K))).astype(np.float32)
    x = f32_to_bf16_torch(rng.integers(-20, 21, (R, T, H)).astype(np.float32))
    _, _, _, h, (recv_x, _, recv_w) = run_oracle_dispatch(topk, E, C, x, w)
    b = brute_handle(topk, E, C)
    yv = rng.integers(-8, 9, size=recv_x.shape).astype(np.float32)
    b0v = rng.integers(-3, 4, (R, T, H)).astype(np.float32)
    b1v = rng.integers(-3, 4, (R, T, H)).astype(np.float32)
    out, out_w = oracle.combine(f32_to_bf16_torch(yv), h, recv_w, bias0=f32_to_bf16_torch(b0v),
                                bias1=f32_to_bf16_torch(b1v), fp32=True)
    exp = b0v.astype(np.float64) + b1v
    for row, (d, s, t) in enumerate(b["triples"]):
        exp[s, t] += yv[row]
    np.testing.assert_array_equal(bf16_to_f64(out), exp)
    np.testing.assert_array_equal(out_w, np.where(topk != -1, w, 0.0).astype(np.float32))

    ll = oracle.ll_dispatch(None, topk, E, T, with_rows=False)
    L, cap = E // R, R * T
    ylv = rng.integers(-6, 7, size=(R, L, cap, H)).astype(np.float32)
    out = oracle.ll_combine(f32_to_bf16_torch(ylv), topk, w, ll["src_info"], ll["layout_range"], E, T,
                            fp32=True)
    lists = brute_ll(topk, E)
    exp = np.zeros((R, T, H))
    for s in range(R):
        for t in range(T):
            for k in range(K):
                e = int(topk[s, t, k])
                if e != -1:
                    exp[s, t] += float(w[s, t, k]) * ylv[e // L, e % L, lists[e].index((s, t))]
    # every term and partial sum is exact in binary32; only the final bf16 rounding acts
    np.testing.assert_array_equal(out, f32_to_bf16_torch(exp.astype(np.float32)))

    m = rng.integers(-1, 5, 11).astype(np.int32)
    gv = rng.integers(-20, 21, (5, 24)).astype(np.float32)
    rv = rng.integers(-20, 21, (11, 24)).astype(np.float32)
    out = oracle.lb_reduce_grads(f32_to_bf16_torch(rv), m, f32_to_bf16_torch(gv), fp32=True)
    exp = gv.astype(np.float64).copy()
    for i in range(11):
        if m[i] >= 0:
            exp[m[i]] += rv[i]
    np.testing.assert_array_equal(bf16_to_f64(out), exp)


def test_fp32_identity_combines_closed_form():
    """Identity experts: f-fold binary32 sums of one bf16 value are exact, so the
    fixed-order combine is bf16(f * x); weights 1/8 give bf16(valid/8 * x)."""
    w_ = synth.WORKLOADS["dsv3"].scaled(num_tokens=40, hidden=64)
    topk = synth.topk_idx(w_)
    x = synth.hidden_rows(w_).view(torch.int16).numpy().view(np.uint16)
    _, _, tin, h, (recv_x, _, _) = run_oracle_dispatch(topk, w_.num_experts, w_.num_channels, x)
    out, _ = oracle.combine(recv_x, h, fp32=True)
    fan = tin.sum(-1).astype(np.float32)
    exp = f32_to_bf16_torch(fan[..., None] * bf16_to_f64(x).astype(np.float32))
    exp[exp == 0x8000] = 0
    np.testing.assert_array_equal(out, exp)

    w_ = synth.WORKLOADS["ll"].scaled(num_tokens=12, hidden=32)
    topk = synth.topk_idx(w_)
    x = synth.hidden_rows(w_).view(torch.int16).numpy().view(np.uint16)
    ll = oracle.ll_dispatch(x, topk, w_.num_experts, w_.tmax)
    out = oracle.ll_combine(ll["packed_recv_x"], topk, np.full(topk.shape, 0.125, np.float32),
                            ll["src_info"], ll["layout_range"], w_.num_experts, w_.tmax, fp32=True)
    exp = f32_to_bf16_torch((topk != -1).sum(-1).astype(np.float32)[..., None] / 8
                            * bf16_to_f64(x).astype(np.float32))
    np.testing.assert_array_equal(out, exp)


def _within_fp32_bound(got, exact, abs_sum, n_terms):
    """|bf16(fp32 sum) - bf16(exact)| <= half a bf16 ulp of each + n * 2^-24 * sum|terms|:
    the recursive-summation error bound (each binary32 operation errs by at most a
    relative 2^-24), plus the two final roundings."""
    def ulp(v):
        a = np.abs(v)
        e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -126.0)
        return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)
    g, r = bf16_to_f64(got), bf16_to_f64(exact)
    tol = 0.5 * ulp(g) + 0.5 * ulp(r) + 1.01 * n_terms * 2.0 ** -24 * bf16_to_f64(abs_sum)
    return np.abs(g - r) <= tol


def test_fp32_reductions_within_the_summation_bound():
    """On random N(0,1) rows the fixed-order results stay within the binary32
    summation error bound of the exact sums (any dropped, doubled or misplaced
    term would break it by a whole term)."""
    w_ = synth.WORKLOADS["dsv3"].scaled(num_tokens=50, hidden=64)
    topk = synth.topk_idx(w_)
    x = synth.hidden_rows(w_).view(torch.int16).numpy().view(np.uint16)
    _, _, _, h, (recv_x, _, _) = run_oracle_dispatch(topk, w_.num_experts, w_.num_channels, x)
    y = synth.expert_rows(w_.seed + 1, recv_x.shape[0], w_.hidden).view(torch.int16).numpy().view(np.uint16)
    b0 = synth.bias_rows(w_, 0).view(torch.int16).numpy().view(np.uint16)
    got, _ = oracle.combine(y, h, bias0=b0, fp32=True)
    exact, _ = oracle.combine(y, h, bias0=b0)
    abs_sum, _ = oracle.combine(y & np.uint16(0x7FFF), h, bias0=b0 & np.uint16(0x7FFF))
    assert _within_fp32_bound(got, exact, abs_sum, 9).all()
    # rows whose large terms cancel: the binary32 sums lose low bits, so the
    # fixed-order result differs from the exact one in places, within the bound
    yw = synth.cancel_rows(w_.seed + 3, recv_x.shape[0], w_.hidden)
    got, _ = oracle.combine(yw, h, fp32=True)
    exact, _ = oracle.combine(yw, h)
    abs_sum, _ = oracle.combine(yw & np.uint16(0x7FFF), h)
    assert _within_fp32_bound(got, exact, abs_sum, 8).all()
    assert (got != exact).mean() > 0.05

    w_ = synth.WORKLOADS["ll"].scaled(num_tokens=20, hidden=64)
    topk = synth.topk_idx(w_)
    wts = synth.topk_weights(w_)
    ll = oracle.ll_dispatch(None, topk, w_.num_experts, w_.tmax, with_rows=False)
    R, L, cap = w_.num_ranks, w_.local_experts, w_.num_ranks * w_.tmax
    y = synth.expert_rows(w_.seed + 2, R * L * cap, w_.hidden).view(torch.int16).numpy().view(np.uint16)
    y = y.reshape(R, L, cap, w_.hidden)
    args = (ll["src_info"], ll["layout_range"], w_.num_experts, w_.tmax)
    got = oracle.ll_combine(y, topk, wts, *args, fp32=True)
    exact = oracle.ll_combine(y, topk, wts, *args)
    abs_sum = oracle.ll_combine(y & np.uint16(0x7FFF), topk, np.abs(wts), *args)
    assert _within_fp32_bound(got, exact, abs_sum, w_.topk).all()

    rng = np.random.default_rng(43)
    m = rng.integers(0, 3, 12).astype(np.int32)
    g = f32_to_bf16_torch(rng.standard_normal((3, 256)).astype(np.float32))
    r = f32_to_bf16_torch(rng.standard_normal((12, 256)).astype(np.float32))
    got = oracle.lb_reduce_grads(r, m, g, fp32=True)
    exact = oracle.lb_reduce_grads(r, m, g)
    abs_sum = oracle.lb_reduce_grads(r & np.uint16(0x7FFF), m, g & np.uint16(0x7FFF))
    assert _within_fp32_bound(got, exact, abs_sum, 13).all()
