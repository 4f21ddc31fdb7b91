"""ep_dispatch_handle_static: the handle build that allocates nothing.

It is meant for callers that cannot call cudaMalloc (device memory fully
reserved by a framework's caching allocator or a serving budget, or code that
must not risk the synchronisation cudaMalloc/cudaFree can cause), so it takes no
context and keeps its scratch in a static device array.  These tests call it
through the C ABI and check that it builds exactly the handle ep_dispatch builds
and the oracle defines, on two calls in a row, and over a run of calls whose
shapes (and so scan tile counts) differ, since the shared scratch keeps the last
call's contents and must be cleared for the next.

This file is collected last on purpose.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth

W = synth.WORKLOADS
HANDLE_OUT = ("send_head", "rank_prefix_matrix", "channel_prefix_matrix",
              "recv_channel_prefix_matrix", "recv_rank_offset", "num_recv_tokens_per_expert")


def static_entry(ep):
    fn = ep.load().ep_dispatch_handle_static
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int32] * 4 + [ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.POINTER(ep.ep_handle), ctypes.c_void_p,
                                          ctypes.c_void_p]
    return fn


def reference_handles(ep, w):
    """(layout on the GPU, ep_dispatch's handle, the oracle's handle) for one workload."""
    R, E, T, C = w.num_ranks, w.num_experts, w.num_tokens, w.num_channels
    topk = synth.topk_idx(w)
    topk_d = torch.from_numpy(topk).cuda()
    x_d = synth.hidden_rows(w).cuda()
    buf = ep.Buffer(R, E, T, w.hidden, w.topk, C)
    ntr, nte, tin = buf.get_dispatch_layout(topk_d)
    _, _, _, ref = buf.dispatch(x_d, topk_d, layout=(ntr, nte, tin))
    assert buf.sync_status() == 0
    buf.destroy()
    _, o_nte, o_tin = oracle.layout(topk, E)
    return (nte, tin), ref, oracle.dispatch_handle(o_tin, o_nte, C, with_src_idx=False)


def static_call(ep, fn, w, nte, tin, err, what):
    R, E, T, C = w.num_ranks, w.num_experts, w.num_tokens, w.num_channels
    h = ep.Handle.empty(R, T, C, E // R, 1, "cuda")
    for name in HANDLE_OUT:
        getattr(h, name).fill_(-7)          # every output must be overwritten
    hs = h.c_struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(R, E, T, C, ctypes.c_void_p(tin.data_ptr()), ctypes.c_void_p(nte.data_ptr()),
            ctypes.byref(hs), ctypes.c_void_p(err.data_ptr()), stream)
    assert rc == 0, f"{what}: status {rc}"
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"{what}: device status {int(err.item())}"
    return h


def check(h, ref, o_ref, what):
    for name in HANDLE_OUT:
        got = getattr(h, name).cpu().numpy()
        np.testing.assert_array_equal(got, getattr(ref, name).cpu().numpy(), err_msg=f"{what}: {name}")
        np.testing.assert_array_equal(got, o_ref[name], err_msg=f"{what}: {name} (oracle)")


CASES = [
    W["tiny"],
    W["dsv3"].scaled(num_tokens=300, hidden=64),
    W["zipf"].scaled(num_tokens=70, hidden=64),
    W["reuse"].scaled(num_tokens=1000, hidden=64),
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_static_handle_matches_ep_dispatch_twice(w):
    import combine_ep_get_11_b200 as ep
    fn = static_entry(ep)
    (nte, tin), ref, o_ref = reference_handles(ep, w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        check(static_call(ep, fn, w, nte, tin, err, f"call {call}"), ref, o_ref, f"call {call}")


@pytest.mark.gpu
def test_static_handle_over_calls_of_changing_shape():
    """Calls whose tile counts differ and do not divide each other, each with its own
    routing: every call must start from cleared scratch, whatever the last left."""
    import combine_ep_get_11_b200 as ep
    fn = static_entry(ep)
    base = W["reuse"].scaled(num_tokens=1000, hidden=64)              # 8000 tokens: 32 tiles
    seq = [base,
           W["zipf"].scaled(num_tokens=70, hidden=64),               # 2240 tokens: 9 tiles, 32 ranks
           W["tiny"],                                                # 128 tokens: 1 tile
           synth.Workload("odd", 3, 9, 610, 16, 4, "uniform_masked", 77, num_channels=7, mask_prob=0.1),
           dataclasses.replace(base, seed=base.seed + 11)]           # the first shape, new routing
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, w in enumerate(seq):
        (nte, tin), ref, o_ref = reference_handles(ep, w)
        check(static_call(ep, fn, w, nte, tin, err, f"call {i} ({w.name})"), ref, o_ref, f"call {i} ({w.name})")


def test_static_handle_rejects_oversized_problem():
    """Sizes beyond the static scratch and missing arguments are refused on the host,
    before any launch."""
    import combine_ep_get_11_b200 as ep
    from combine_ep_get_11_b200 import build
    build.build()
    fn = static_entry(ep)
    dummy = ctypes.c_void_p(256)            # never dereferenced: the checks come first
    hs = ep.ep_handle(*([dummy] * 8))
    # 32 ranks x 65536 tokens needs 2 MiB of tile flags alone
    assert fn(32, 256, 65536, 10, dummy, dummy, ctypes.byref(hs), dummy, None) == 3
    # 32 ranks x 8192 tokens needs 270,592 bytes: within the 512 KiB array (refused here
    # only for the missing error word, before any launch)
    assert fn(32, 256, 8192, 10, dummy, dummy, ctypes.byref(hs), None, None) == 1
    # bad shapes are argument errors
    assert fn(0, 8, 10, 4, dummy, dummy, ctypes.byref(hs), dummy, None) == 1
    assert fn(4, 10, 10, 4, dummy, dummy, ctypes.byref(hs), dummy, None) == 1
