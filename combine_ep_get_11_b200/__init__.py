"""Python binding of libep.so: MoE dispatch / combine on virtual EP ranks (B200).

Argument marshalling only.  Every step of the path runs in the library (its CUDA
kernels, and its host code for the receive count); torch supplies device memory
and the current stream.  The entry points keep the C names (``ep_create``,
``ep_get_dispatch_layout``, ``ep_get_num_recv``, ``ep_dispatch``,
``ep_dispatch_cached``, ``ep_combine``, ``ep_ll_dispatch``, ``ep_ll_combine``,
``ep_sync_status``); ``Buffer`` wraps them with output allocation, in the shape
of DeepEP's ``Buffer`` API.  There is no CPU fallback: if the library is
missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libep.so")

EP_OK = 0
STATUS_NAMES = {0: "EP_OK", 1: "EP_ERR_INVALID_ARG", 2: "EP_ERR_ALIGNMENT", 3: "EP_ERR_CAPACITY",
                4: "EP_ERR_BAD_TOPK", 5: "EP_ERR_HANDLE_MISMATCH", 6: "EP_ERR_TIMEOUT",
                7: "EP_ERR_CUDA", 8: "EP_ERR_UNIMPLEMENTED"}
PROFILE_KINDS = ["layout", "scan", "dispatch", "dispatch_cached", "combine", "ll_count",
                 "ll_copy", "ll_combine", "ll_copy_fp8", "lb_prefetch", "lb_reduce"]

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


class EpError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}" + (f" ({detail})" if detail else ""))


class ep_config(ctypes.Structure):
    _fields_ = [("num_ranks", _i32), ("num_experts", _i32), ("num_tokens", _i32),
                ("hidden", _i32), ("topk", _i32), ("num_channels", _i32),
                ("ll_max_tokens_per_rank", _i32)]


class ep_handle(ctypes.Structure):
    _fields_ = [("rank_prefix_matrix", _vp), ("channel_prefix_matrix", _vp),
                ("recv_channel_prefix_matrix", _vp), ("recv_src_idx", _vp),
                ("is_token_in_rank", _vp), ("send_head", _vp), ("recv_rank_offset", _vp),
                ("num_recv_tokens_per_expert", _vp)]


class ep_handle_sizes(ctypes.Structure):
    _fields_ = [(n, _i64) for n in (
        "rank_prefix_matrix", "channel_prefix_matrix", "recv_channel_prefix_matrix",
        "recv_src_idx_max", "is_token_in_rank", "send_head", "recv_rank_offset",
        "num_recv_tokens_per_expert", "ll_packed_recv_x", "ll_packed_recv_count",
        "ll_src_info", "ll_layout_range")]


# name -> (restype, argtypes); the exported C ABI, mirrored from include/ep.h
_SIGNATURES = {
    "ep_create": (ctypes.c_int, [ctypes.POINTER(ep_config), ctypes.POINTER(_vp)]),
    "ep_destroy": (ctypes.c_int, [_vp]),
    "ep_workspace_bytes": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_size_t)]),
    "ep_handle_layout": (ctypes.c_int, [_vp, ctypes.POINTER(ep_handle_sizes)]),
    "ep_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ep_last_error": (ctypes.c_char_p, [_vp]),
    "ep_sync_status": (ctypes.c_int, [_vp, _vp]),
    "ep_kernel_launch_count": (ctypes.c_uint64, []),
    "ep_test_offset_tickets": (ctypes.c_int, [_vp, _i64]),
    "ep_check_handle": (ctypes.c_int, [_vp, _vp, ctypes.POINTER(ep_handle), _vp, _vp]),
    "ep_get_dispatch_layout": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ep_dispatch": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(ep_handle),
                                   _vp, _vp, _vp, _i64, ctypes.POINTER(_i64), _vp, _vp]),
    "ep_get_num_recv": (ctypes.c_int, [_vp, _vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64), _vp, _vp]),
    "ep_dispatch_cached": (ctypes.c_int, [_vp, _vp, ctypes.POINTER(ep_handle), _vp, _i64, _vp, _vp]),
    "ep_combine": (ctypes.c_int, [_vp, _vp, _i64, ctypes.POINTER(ep_handle), _vp, _vp, _vp, _vp,
                                  _vp, _vp, _vp]),
    "ep_ll_dispatch": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ep_ll_dispatch_fp8": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ep_ll_combine": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ep_lb_prefetch_weights": (ctypes.c_int, [_vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp]),
    "ep_lb_reduce_grads": (ctypes.c_int, [_vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp]),
    "ep_ll_update_mask": (ctypes.c_int, [_vp, _i32, _i32, _vp]),
    "ep_ll_query_mask": (ctypes.c_int, [_vp, _vp, _vp]),
    "ep_ll_clean_mask": (ctypes.c_int, [_vp, _vp]),
    "ep_create_sharded": (ctypes.c_int, [ctypes.POINTER(ep_config), ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(_vp)]),
    "ep_sharded_handle": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ep_sharded_dispatch": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.POINTER(_vp),
                                           ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                           _i64, _vp, _vp]),
    "ep_sharded_combine": (ctypes.c_int, [_vp, ctypes.c_int, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i64,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ep_shared_alloc": (ctypes.c_int, [ctypes.c_size_t, ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_uint8)]),
    "ep_shared_free": (ctypes.c_int, [_vp]),
    "ep_ipc_open": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(_vp)]),
    "ep_ipc_close": (ctypes.c_int, [_vp]),
    "ep_profile_enable": (ctypes.c_int, [_vp, ctypes.c_int]),
    "ep_profile_read": (ctypes.c_int, [_vp, ctypes.POINTER(_i64), ctypes.POINTER(ctypes.c_double)]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libep.so (built by combine_ep_get_11_b200.build).  Raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m combine_ep_get_11_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _event(ev):
    return None if ev is None else ctypes.c_void_p(ev.cuda_event)


def _check(rc: int, what: str, ctx=None):
    if rc != EP_OK:
        detail = load().ep_last_error(ctx).decode() if ctx else ""
        raise EpError(rc, what, detail)


def kernel_launch_count() -> int:
    return int(load().ep_kernel_launch_count())


# ---------------------------------------------------------------- raw entries

def ep_create(num_ranks, num_experts, num_tokens, hidden, topk, num_channels=10,
              ll_max_tokens_per_rank=0):
    cfg = ep_config(num_ranks, num_experts, num_tokens, hidden, topk, num_channels,
                    ll_max_tokens_per_rank)
    out = _vp()
    _check(load().ep_create(ctypes.byref(cfg), ctypes.byref(out)), "ep_create")
    return out


def ep_destroy(ctx):
    _check(load().ep_destroy(ctx), "ep_destroy")


def ep_sync_status(ctx, stream=None) -> int:
    """Synchronize and return the device status code (0 = OK) without raising."""
    return load().ep_sync_status(ctx, _stream(stream))


@dataclasses.dataclass
class Handle:
    """Device arrays of one dispatch handle (see ep_handle in include/ep.h)."""
    rank_prefix_matrix: torch.Tensor
    channel_prefix_matrix: torch.Tensor
    recv_channel_prefix_matrix: torch.Tensor
    recv_src_idx: torch.Tensor
    is_token_in_rank: torch.Tensor
    send_head: torch.Tensor
    recv_rank_offset: torch.Tensor
    num_recv_tokens_per_expert: torch.Tensor
    num_recv_rows: int = -1

    def c_struct(self) -> ep_handle:
        return ep_handle(*[_ptr(getattr(self, f.name)) for f in dataclasses.fields(self)
                           if f.name != "num_recv_rows"])

    @staticmethod
    def empty(R, T, C, L, recv_capacity, device):
        i32 = dict(dtype=torch.int32, device=device)
        return Handle(
            rank_prefix_matrix=torch.empty((R, R), **i32),
            channel_prefix_matrix=torch.empty((R, R, C), **i32),
            recv_channel_prefix_matrix=torch.empty((R, R, C), **i32),
            recv_src_idx=torch.empty((max(recv_capacity, 1),), **i32),
            is_token_in_rank=torch.empty((R, T, R), dtype=torch.uint8, device=device),
            send_head=torch.empty((R, T, R), **i32),
            recv_rank_offset=torch.empty((R + 1,), dtype=torch.int64, device=device),
            num_recv_tokens_per_expert=torch.empty((R, L), **i32),
        )


def ep_get_dispatch_layout(ctx, topk_idx, num_tokens_per_rank, num_tokens_per_expert,
                           is_token_in_rank, stream=None, wait_event=None):
    _check(load().ep_get_dispatch_layout(ctx, _ptr(topk_idx), _ptr(num_tokens_per_rank),
                                         _ptr(num_tokens_per_expert), _ptr(is_token_in_rank),
                                         _stream(stream), _event(wait_event)),
           "ep_get_dispatch_layout", ctx)


def ep_dispatch(ctx, x, topk_idx, topk_weights, num_tokens_per_rank, num_tokens_per_expert,
                is_token_in_rank, handle: Handle, recv_x, recv_topk_idx, recv_topk_weights,
                recv_capacity_rows, want_num_recv=False, stream=None, wait_event=None):
    n = _i64(-1)
    hs = handle.c_struct()
    _check(load().ep_dispatch(ctx, _ptr(x), _ptr(topk_idx), _ptr(topk_weights),
                              _ptr(num_tokens_per_rank), _ptr(num_tokens_per_expert),
                              _ptr(is_token_in_rank), ctypes.byref(hs), _ptr(recv_x),
                              _ptr(recv_topk_idx), _ptr(recv_topk_weights), recv_capacity_rows,
                              ctypes.byref(n) if want_num_recv else None,
                              _stream(stream), _event(wait_event)), "ep_dispatch", ctx)
    return int(n.value) if want_num_recv else None


def ep_get_num_recv(ctx, num_tokens_per_rank, num_ranks: int, stream=None, wait_event=None):
    """(N, [N_0 .. N_{R-1}]): receive rows in all and per destination rank, from the
    layout's per-rank counts (one host synchronisation, inside the library)."""
    n = _i64(-1)
    per = (_i64 * num_ranks)()
    _check(load().ep_get_num_recv(ctx, _ptr(num_tokens_per_rank), ctypes.byref(n), per, _stream(stream),
                                  _event(wait_event)), "ep_get_num_recv", ctx)
    return int(n.value), [int(v) for v in per]


def ep_dispatch_cached(ctx, x, handle: Handle, recv_x, recv_capacity_rows, stream=None,
                       wait_event=None):
    hs = handle.c_struct()
    _check(load().ep_dispatch_cached(ctx, _ptr(x), ctypes.byref(hs), _ptr(recv_x),
                                     recv_capacity_rows, _stream(stream), _event(wait_event)),
           "ep_dispatch_cached", ctx)


def ep_combine(ctx, y, num_recv_rows, handle: Handle, recv_topk_weights, bias0, bias1, out_x,
               out_topk_weights, stream=None, wait_event=None):
    hs = handle.c_struct()
    _check(load().ep_combine(ctx, _ptr(y), num_recv_rows, ctypes.byref(hs), _ptr(recv_topk_weights),
                             _ptr(bias0), _ptr(bias1), _ptr(out_x), _ptr(out_topk_weights),
                             _stream(stream), _event(wait_event)), "ep_combine", ctx)


def ep_ll_dispatch(ctx, x, topk_idx, packed_recv_x, packed_recv_count, src_info, layout_range,
                   stream=None, wait_event=None):
    _check(load().ep_ll_dispatch(ctx, _ptr(x), _ptr(topk_idx), _ptr(packed_recv_x),
                                 _ptr(packed_recv_count), _ptr(src_info), _ptr(layout_range),
                                 _stream(stream), _event(wait_event)), "ep_ll_dispatch", ctx)


def ep_ll_dispatch_fp8(ctx, x, topk_idx, packed_recv_x_fp8, packed_recv_scales, packed_recv_count,
                       src_info, layout_range, stream=None, wait_event=None):
    _check(load().ep_ll_dispatch_fp8(ctx, _ptr(x), _ptr(topk_idx), _ptr(packed_recv_x_fp8),
                                     _ptr(packed_recv_scales), _ptr(packed_recv_count), _ptr(src_info),
                                     _ptr(layout_range), _stream(stream), _event(wait_event)),
           "ep_ll_dispatch_fp8", ctx)


def ep_ll_combine(ctx, y, topk_idx, topk_weights, src_info, layout_range, out_x, stream=None,
                  wait_event=None):
    _check(load().ep_ll_combine(ctx, _ptr(y), _ptr(topk_idx), _ptr(topk_weights), _ptr(src_info),
                                _ptr(layout_range), _ptr(out_x), _stream(stream),
                                _event(wait_event)), "ep_ll_combine", ctx)


def ep_lb_prefetch_weights(ctx, expert_weights, redundancy_mapping, redundant_weights, stream=None,
                           wait_event=None):
    """expert_weights [E, ...] bf16, redundancy_mapping [N] int32, redundant_weights [N, ...] bf16."""
    w = expert_weights[0].numel() if expert_weights.dim() > 1 else 1
    _check(load().ep_lb_prefetch_weights(ctx, _ptr(expert_weights), w, _ptr(redundancy_mapping),
                                         redundancy_mapping.numel(), _ptr(redundant_weights),
                                         _stream(stream), _event(wait_event)), "ep_lb_prefetch_weights", ctx)


def ep_lb_reduce_grads(ctx, redundant_grads, redundancy_mapping, expert_grads, stream=None, wait_event=None):
    """redundant_grads [N, ...] bf16, redundancy_mapping [N] int32, expert_grads [E, ...] bf16 (in/out)."""
    w = expert_grads[0].numel() if expert_grads.dim() > 1 else 1
    _check(load().ep_lb_reduce_grads(ctx, _ptr(redundant_grads), w, _ptr(redundancy_mapping),
                                     redundancy_mapping.numel(), _ptr(expert_grads), _stream(stream),
                                     _event(wait_event)), "ep_lb_reduce_grads", ctx)


def ep_ll_update_mask(ctx, rank: int, masked: bool, stream=None):
    _check(load().ep_ll_update_mask(ctx, rank, int(bool(masked)), _stream(stream)), "ep_ll_update_mask", ctx)


def ep_ll_query_mask(ctx, out, stream=None):
    """out: CPU int32 tensor [R]; filled with 0 (active) / 1 (masked)."""
    assert out.device.type == "cpu" and out.dtype == torch.int32 and out.is_contiguous()
    _check(load().ep_ll_query_mask(ctx, ctypes.c_void_p(out.data_ptr()), _stream(stream)),
           "ep_ll_query_mask", ctx)
    return out


def ep_ll_clean_mask(ctx, stream=None):
    _check(load().ep_ll_clean_mask(ctx, _stream(stream)), "ep_ll_clean_mask", ctx)


def ep_profile_enable(ctx, enable: bool = True):
    _check(load().ep_profile_enable(ctx, int(enable)), "ep_profile_enable", ctx)


def ep_profile_read(ctx) -> dict:
    n = (_i64 * len(PROFILE_KINDS))()
    ms = (ctypes.c_double * len(PROFILE_KINDS))()
    _check(load().ep_profile_read(ctx, n, ms), "ep_profile_read", ctx)
    return {k: (int(n[i]), float(ms[i])) for i, k in enumerate(PROFILE_KINDS)}


# ---------------------------------------------------------- convenience API

_deferred: list = []     # contexts whose release waits for the end of a graph capture


def _release_deferred():
    if not _deferred or (torch.cuda.is_available() and torch.cuda.is_current_stream_capturing()):
        return
    while _deferred:
        ep_destroy(_deferred.pop())


class Buffer:
    """Dispatch/combine on R virtual ranks of one GPU, shaped like DeepEP's Buffer.

    Inputs are stacked over ranks: x [R, T, H] bf16, topk_idx [R, T, K] int64,
    topk_weights [R, T, K] float32, all on this GPU.
    """

    def __init__(self, num_ranks, num_experts, num_tokens, hidden, topk, num_channels=10,
                 ll_max_tokens_per_rank=0, device=None):
        self.device = (torch.device("cuda", torch.cuda.current_device()) if device is None
                       else torch.device(device))
        _release_deferred()
        with torch.cuda.device(self.device):
            self.ctx = ep_create(num_ranks, num_experts, num_tokens, hidden, topk, num_channels,
                                 ll_max_tokens_per_rank)
        self.R, self.E, self.T, self.H, self.K, self.C = (num_ranks, num_experts, num_tokens, hidden,
                                                          topk, num_channels)
        self.L = num_experts // num_ranks
        self.Tmax = ll_max_tokens_per_rank or num_tokens

    def destroy(self):
        _release_deferred()
        if self.ctx is not None:
            ep_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        # The garbage collector may run this in the middle of a CUDA graph capture,
        # where freeing device memory would invalidate the capture: the context is
        # then released by the next Buffer created or destroyed outside a capture.
        try:
            if self.ctx is None:
                return
            if torch.cuda.is_available() and torch.cuda.is_current_stream_capturing():
                _deferred.append(self.ctx)
                self.ctx = None
            else:
                self.destroy()
        except Exception:
            pass

    def sizes(self) -> ep_handle_sizes:
        s = ep_handle_sizes()
        _check(load().ep_handle_layout(self.ctx, ctypes.byref(s)), "ep_handle_layout", self.ctx)
        return s

    def sync_status(self, stream=None) -> int:
        return ep_sync_status(self.ctx, stream)

    def check(self, stream=None):
        rc = ep_sync_status(self.ctx, stream)
        _check(rc, "device status", self.ctx)

    def get_dispatch_layout(self, topk_idx, stream=None):
        ntr = torch.empty((self.R, self.R), dtype=torch.int32, device=self.device)
        nte = torch.empty((self.R, self.E), dtype=torch.int32, device=self.device)
        tin = torch.empty((self.R, self.T, self.R), dtype=torch.uint8, device=self.device)
        ep_get_dispatch_layout(self.ctx, topk_idx, ntr, nte, tin, stream)
        return ntr, nte, tin

    def dispatch(self, x, topk_idx, topk_weights=None, layout=None, recv_capacity=None, stream=None):
        """Returns (recv_x [N,H], recv_topk_idx [N,K], recv_topk_weights [N,K] or None, handle).

        Without recv_capacity the receive size is learned from the layout with one
        host read (the pages' CPU-GPU synchronisation); with it, nothing blocks."""
        if layout is None:
            layout = self.get_dispatch_layout(topk_idx, stream)
        ntr, nte, tin = layout
        if recv_capacity is None:
            recv_capacity, _ = ep_get_num_recv(self.ctx, ntr, self.R, stream)
        handle = Handle.empty(self.R, self.T, self.C, self.L, recv_capacity, self.device)
        handle.is_token_in_rank = tin
        recv_x = torch.empty((recv_capacity, self.H), dtype=torch.bfloat16, device=self.device)
        recv_idx = torch.empty((recv_capacity, self.K), dtype=torch.int64, device=self.device)
        recv_w = None if topk_weights is None else torch.empty((recv_capacity, self.K),
                                                               dtype=torch.float32, device=self.device)
        ep_dispatch(self.ctx, x, topk_idx, topk_weights, ntr, nte, tin, handle,
                    recv_x if recv_capacity else None, recv_idx if recv_capacity else None,
                    recv_w if recv_capacity else None, recv_capacity, stream=stream)
        handle.num_recv_rows = recv_capacity
        return recv_x, recv_idx, recv_w, handle

    def check_handle(self, topk_idx, handle: Handle, stream=None) -> bool:
        """True if `handle` is the dispatch handle of this routing (the reuse
        contract); synchronizes the stream to read the result."""
        hs = handle.c_struct()
        _check(load().ep_check_handle(self.ctx, _ptr(topk_idx), ctypes.byref(hs), _stream(stream), None),
               "ep_check_handle", self.ctx)
        rc = ep_sync_status(self.ctx, stream)
        if rc not in (EP_OK, 5):
            _check(rc, "device status", self.ctx)
        return rc == EP_OK

    def dispatch_cached(self, x, handle: Handle, stream=None):
        recv_x = torch.empty((handle.num_recv_rows, self.H), dtype=torch.bfloat16, device=self.device)
        ep_dispatch_cached(self.ctx, x, handle, recv_x, handle.num_recv_rows, stream)
        return recv_x

    def combine(self, y, handle: Handle, recv_topk_weights=None, bias=(None, None), stream=None):
        out = torch.empty((self.R, self.T, self.H), dtype=torch.bfloat16, device=self.device)
        out_w = None if recv_topk_weights is None else torch.empty(
            (self.R, self.T, self.K), dtype=torch.float32, device=self.device)
        ep_combine(self.ctx, y, y.shape[0], handle, recv_topk_weights, bias[0], bias[1], out, out_w,
                   stream)
        return out, out_w

    def low_latency_dispatch(self, x, topk_idx, use_fp8=False, stream=None):
        """Returns (packed, count, handle); with use_fp8, packed is (codes u8, scales f32)."""
        cap = self.R * self.Tmax
        count = torch.empty((self.R, self.L), dtype=torch.int32, device=self.device)
        src_info = torch.empty((self.R, self.L, cap), dtype=torch.int32, device=self.device)
        layout_range = torch.empty((self.R, self.L, self.R, 2), dtype=torch.int32, device=self.device)
        if use_fp8:
            codes = torch.empty((self.R, self.L, cap, self.H), dtype=torch.uint8, device=self.device)
            scales = torch.empty((self.R, self.L, cap, self.H // 128), dtype=torch.float32, device=self.device)
            ep_ll_dispatch_fp8(self.ctx, x, topk_idx, codes, scales, count, src_info, layout_range, stream)
            return (codes, scales), count, (src_info, layout_range)
        packed = torch.empty((self.R, self.L, cap, self.H), dtype=torch.bfloat16, device=self.device)
        ep_ll_dispatch(self.ctx, x, topk_idx, packed, count, src_info, layout_range, stream)
        return packed, count, (src_info, layout_range)

    def lb_prefetch_weights(self, redundant_expert_weights, expert_weights, redundancy_mapping, stream=None):
        ep_lb_prefetch_weights(self.ctx, expert_weights, redundancy_mapping, redundant_expert_weights, stream)

    def lb_reduce_grads(self, redundant_expert_grads, expert_grads, redundancy_mapping, stream=None):
        ep_lb_reduce_grads(self.ctx, redundant_expert_grads, redundancy_mapping, expert_grads, stream)

    def low_latency_update_mask_buffer(self, rank_to_mask: int, mask: bool = True, stream=None):
        ep_ll_update_mask(self.ctx, rank_to_mask, mask, stream)

    def low_latency_query_mask_buffer(self, out=None, stream=None):
        out = torch.empty(self.R, dtype=torch.int32) if out is None else out
        return ep_ll_query_mask(self.ctx, out, stream)

    def low_latency_clean_mask_buffer(self, stream=None):
        ep_ll_clean_mask(self.ctx, stream)

    def low_latency_combine(self, y, topk_idx, topk_weights, ll_handle, stream=None):
        out = torch.empty((self.R, self.T, self.H), dtype=torch.bfloat16, device=self.device)
        src_info, layout_range = ll_handle
        ep_ll_combine(self.ctx, y, topk_idx, topk_weights, src_info, layout_range, out, stream)
        return out
