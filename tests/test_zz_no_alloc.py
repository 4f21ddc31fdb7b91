"""ep_dispatch_handle_static: the handle build that allocates nothing.

It is meant for callers that cannot call cudaMalloc (device memory fully
reserved by a framework's caching allocator or a serving budget, or code that
must not risk the synchronisation cudaMalloc/cudaFree can cause), so it takes no
context and keeps its scratch in a static device array.  These tests call it
through the C ABI and check that it builds exactly the handle ep_dispatch builds,
on two calls in a row (the shared scratch must be cleared between calls).

This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

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
    R, E, T, C = w.num_ranks, w.num_experts, w.num_tokens, w.num_channels
    topk_d = torch.from_numpy(synth.topk_idx(w)).cuda()
    x_d = synth.hidden_rows(w).cuda()
    buf = ep.Buffer(R, E, T, w.hidden, w.topk, C)
    ntr, nte, tin = buf.get_dispatch_layout(topk_d)
    _, _, _, ref = buf.dispatch(x_d, topk_d, layout=(ntr, nte, tin))
    assert buf.sync_status() == 0

    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        h = ep.Handle.empty(R, T, C, E // R, 1, "cuda")
        for name in HANDLE_OUT:
            getattr(h, name).fill_(-7)          # every output must be overwritten
        hs = h.c_struct()
        rc = fn(R, E, T, C, ctypes.c_void_p(tin.data_ptr()), ctypes.c_void_p(nte.data_ptr()),
                ctypes.byref(hs), ctypes.c_void_p(err.data_ptr()), stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        for name in HANDLE_OUT:
            np.testing.assert_array_equal(getattr(h, name).cpu().numpy(),
                                          getattr(ref, name).cpu().numpy(),
                                          err_msg=f"call {call}: {name}")
        assert int(err.item()) == 0
    buf.destroy()


def test_static_handle_rejects_oversized_problem():
    """Sizes beyond the static scratch are refused on the host, before any launch."""
    import combine_ep_get_11_b200 as ep
    from combine_ep_get_11_b200 import build
    build.build()
    fn = static_entry(ep)
    dummy = ctypes.c_void_p(256)            # never dereferenced: the size check comes first
    hs = ep.ep_handle(*([dummy] * 8))
    # 32 ranks x 65536 tokens needs 2 MiB of tile flags alone
    assert fn(32, 256, 65536, 10, dummy, dummy, ctypes.byref(hs), None, None) == 3
    # bad shapes are argument errors
    assert fn(0, 8, 10, 4, dummy, dummy, ctypes.byref(hs), None, None) == 1
    assert fn(4, 10, 10, 4, dummy, dummy, ctypes.byref(hs), None, None) == 1
