"""Python face of the CPU oracle (numpy in, numpy out).

TEST INFRASTRUCTURE ONLY.  The oracle is a plain, slow, single-threaded CPU
statement of the dispatch/combine hot path (ep_oracle.cpp).  Only the tests,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg use it; the
CUDA library and its Python binding never import it.

Arrays are numpy; bf16 tensors travel as ``np.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_c_i32 = ctypes.c_int32
_c_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p

OK, BAD_ARG, BAD_TOPK, CAPACITY, NOT_FOUND = 0, 1, 2, 3, 4


class OracleError(RuntimeError):
    pass


def load_library(path: str):
    """Load an oracle build from `path` and declare its C signatures."""
    L = ctypes.CDLL(path)
    L.oracle_round_bf16.argtypes = [_ptr, _ptr, _c_i64]
    L.oracle_round_bf16.restype = None
    L.oracle_layout.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _ptr, _ptr, _ptr, _ptr]
    L.oracle_dispatch_handle.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _ptr, _ptr,
                                             _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _c_i64]
    L.oracle_dispatch_rows.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                           _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr]
    L.oracle_combine.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _ptr, _c_i64, _ptr, _ptr,
                                     _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _c_i64]
    L.oracle_combine_fp32.argtypes = L.oracle_combine.argtypes
    L.oracle_ll_dispatch.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                         _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr]
    L.oracle_ll_combine.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                        _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _c_i64, _ptr]
    L.oracle_ll_combine_fp32.argtypes = L.oracle_ll_combine.argtypes
    L.oracle_fp8_e4m3_encode.argtypes = [_ptr, _ptr, _c_i64]
    L.oracle_fp8_e4m3_encode.restype = None
    L.oracle_quantize_e4m3_blocks.argtypes = [_ptr, _c_i64, _c_i32, _c_i32, _ptr, _ptr]
    L.oracle_lb_prefetch_weights.argtypes = [_ptr, _c_i32, _c_i64, _ptr, _c_i32, _ptr]
    L.oracle_lb_reduce_grads.argtypes = [_ptr, _ptr, _c_i32, _ptr, _c_i32, _c_i64]
    L.oracle_lb_reduce_grads_fp32.argtypes = L.oracle_lb_reduce_grads.argtypes
    for name in ("oracle_layout", "oracle_dispatch_handle", "oracle_dispatch_rows",
                 "oracle_combine", "oracle_combine_fp32", "oracle_ll_dispatch", "oracle_ll_combine",
                 "oracle_ll_combine_fp32", "oracle_quantize_e4m3_blocks", "oracle_lb_prefetch_weights",
                 "oracle_lb_reduce_grads", "oracle_lb_reduce_grads_fp32"):
        getattr(L, name).restype = ctypes.c_int
    return L


def lib():
    """The oracle library (EP_ORACLE_LIB may name another build, e.g. a planted mutant)."""
    global _LIB
    if _LIB is None:
        _LIB = load_library(os.environ.get("EP_ORACLE_LIB") or _build.build())
    return _LIB


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != OK:
        raise OracleError(f"{what} failed with oracle status {rc}")


def round_bf16(values: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_round_bf16(_p(v), _p(out), v.size)
    return out


def layout(topk_idx: np.ndarray, num_experts: int):
    """topk_idx [R, T, K] int64 -> (num_tokens_per_rank [R,R], num_tokens_per_expert [R,E],
    is_token_in_rank [R,T,R] u8)."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    R, T, K = topk_idx.shape
    ntr = np.empty((R, R), np.int32)
    nte = np.empty((R, num_experts), np.int32)
    tin = np.empty((R, T, R), np.uint8)
    _check(lib().oracle_layout(R, num_experts, T, K, _p(topk_idx), _p(ntr), _p(nte), _p(tin)),
           "oracle_layout")
    return ntr, nte, tin


def dispatch_handle(is_token_in_rank: np.ndarray, num_tokens_per_expert: np.ndarray,
                    num_channels: int, with_src_idx: bool = True):
    """Handle matrices.  Returns a dict of numpy arrays."""
    tin = np.ascontiguousarray(is_token_in_rank, dtype=np.uint8)
    nte = np.ascontiguousarray(num_tokens_per_expert, dtype=np.int32)
    R, T, _ = tin.shape
    E = nte.shape[1]
    L = E // R
    C = num_channels
    h = {
        "rank_prefix_matrix": np.empty((R, R), np.int32),
        "channel_prefix_matrix": np.empty((R, R, C), np.int32),
        "recv_channel_prefix_matrix": np.empty((R, R, C), np.int32),
        "send_head": np.empty((R, T, R), np.int32),
        "recv_rank_offset": np.empty((R + 1,), np.int64),
        "num_recv_tokens_per_expert": np.empty((R, L), np.int32),
    }
    cap = int(tin.astype(np.int64).sum())
    src = np.empty((max(cap, 1),), np.int32) if with_src_idx else None
    _check(lib().oracle_dispatch_handle(
        R, E, T, C, _p(tin), _p(nte), _p(h["rank_prefix_matrix"]), _p(h["channel_prefix_matrix"]),
        _p(h["recv_channel_prefix_matrix"]), _p(h["send_head"]), _p(h["recv_rank_offset"]),
        _p(h["num_recv_tokens_per_expert"]), _p(src), cap), "oracle_dispatch_handle")
    if with_src_idx:
        h["recv_src_idx"] = src[:cap].copy()
    h["is_token_in_rank"] = tin
    return h


def dispatch_rows(x, topk_idx: np.ndarray, topk_weights, handle: dict, num_experts: int):
    """x [R,T,H] uint16 (bf16 bits) -> recv_x [N,H] u16, recv_topk_idx [N,K] i64,
    recv_topk_weights [N,K] f32 (None if topk_weights is None).  With x=None only the
    top-k rows are produced (recv_x is None)."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    R, T, K = topk_idx.shape
    N = int(handle["recv_rank_offset"][-1])
    if x is not None:
        x = np.ascontiguousarray(x, dtype=np.uint16)
        H = x.shape[2]
        recv_x = np.empty((N, H), np.uint16)
    else:
        H = 1
        recv_x = None
    recv_idx = np.empty((N, K), np.int64)
    w = None if topk_weights is None else np.ascontiguousarray(topk_weights, dtype=np.float32)
    recv_w = None if w is None else np.empty((N, K), np.float32)
    _check(lib().oracle_dispatch_rows(
        R, num_experts, T, K, H, _p(x), _p(topk_idx), _p(w), _p(handle["send_head"]),
        _p(handle["recv_rank_offset"]), _p(recv_x), _p(recv_idx), _p(recv_w)),
        "oracle_dispatch_rows")
    return recv_x, recv_idx, recv_w


def combine(y: np.ndarray, handle: dict, recv_topk_weights=None, bias0=None, bias1=None,
            tokens=None, topk: int | None = None, fp32: bool = False):
    """y [N,H] u16 -> (out_x [R,T,H] u16 or [n,H] for a token list, out_w or None).

    fp32=False: the exact sum (fp64 accumulation, one bf16 rounding).
    fp32=True: the fixed-order fp32 definition (ascending destination rank, then
    the biases; binary32 additions from +0, one bf16 rounding)."""
    y = np.ascontiguousarray(y, dtype=np.uint16)
    sh = handle["send_head"]
    R, T, _ = sh.shape
    H = y.shape[1]
    if recv_topk_weights is not None:
        rw = np.ascontiguousarray(recv_topk_weights, dtype=np.float32)
        K = rw.shape[1]
    else:
        rw = None
        K = topk if topk is not None else 1
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = R * T if tok is None else tok.size
    out = np.empty((n, H), np.uint16)
    out_w = np.empty((n, K), np.float32) if rw is not None else None
    b0 = None if bias0 is None else np.ascontiguousarray(bias0, dtype=np.uint16)
    b1 = None if bias1 is None else np.ascontiguousarray(bias1, dtype=np.uint16)
    fn = lib().oracle_combine_fp32 if fp32 else lib().oracle_combine
    _check(fn(
        R, T, K, H, _p(y), y.shape[0], _p(sh), _p(handle["recv_rank_offset"]), _p(rw),
        _p(b0), _p(b1), _p(out), _p(out_w), _p(tok), 0 if tok is None else tok.size),
        "oracle_combine" + ("_fp32" if fp32 else ""))
    if tok is None:
        out = out.reshape(R, T, H)
        if out_w is not None:
            out_w = out_w.reshape(R, T, K)
    return out, out_w


def _mask(rank_mask, R):
    if rank_mask is None:
        return None
    m = np.ascontiguousarray(rank_mask, dtype=np.int32)
    assert m.shape == (R,)
    return m


def ll_dispatch(x, topk_idx, num_experts: int, max_tokens_per_rank: int, with_rows: bool = True,
                rank_mask=None):
    """Returns dict with packed_recv_x [R,L,R*Tmax,H] (if with_rows), packed_recv_count [R,L],
    src_info [R,L,R*Tmax], layout_range [R,L,R,2]."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    R, T, K = topk_idx.shape
    x = np.ascontiguousarray(x, dtype=np.uint16) if x is not None else None
    H = x.shape[2] if x is not None else 1
    L = num_experts // R
    cap = R * max_tokens_per_rank
    packed = np.zeros((R, L, cap, H), np.uint16) if with_rows else None
    count = np.empty((R, L), np.int32)
    src_info = np.full((R, L, cap), -1, np.int32)
    layout_range = np.empty((R, L, R, 2), np.int32)
    m = _mask(rank_mask, R)
    _check(lib().oracle_ll_dispatch(
        R, num_experts, T, K, H, max_tokens_per_rank, _p(x), _p(topk_idx), _p(packed),
        _p(count), _p(src_info), _p(layout_range), _p(m)), "oracle_ll_dispatch")
    return {"packed_recv_x": packed, "packed_recv_count": count, "src_info": src_info,
            "layout_range": layout_range}


def ll_combine(y, topk_idx, topk_weights, src_info, layout_range, num_experts: int,
               max_tokens_per_rank: int, tokens=None, rank_mask=None, fp32: bool = False):
    """Weighted low-latency combine.  fp32=False: the exact sum (fp64, one bf16
    rounding); fp32=True: the fixed-order definition (binary32 fused multiply-add
    chain from +0 over ascending (expert id, k), one bf16 rounding)."""
    y = np.ascontiguousarray(y, dtype=np.uint16)
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int64)
    w = np.ascontiguousarray(topk_weights, dtype=np.float32)
    R, T, K = topk_idx.shape
    H = y.shape[-1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = R * T if tok is None else tok.size
    out = np.empty((n, H), np.uint16)
    fn = lib().oracle_ll_combine_fp32 if fp32 else lib().oracle_ll_combine
    _check(fn(
        R, num_experts, T, K, H, max_tokens_per_rank, _p(y), _p(topk_idx), _p(w),
        _p(np.ascontiguousarray(src_info, dtype=np.int32)),
        _p(np.ascontiguousarray(layout_range, dtype=np.int32)), _p(out), _p(tok),
        0 if tok is None else tok.size, _p(_mask(rank_mask, R))),
        "oracle_ll_combine" + ("_fp32" if fp32 else ""))
    return out.reshape(R, T, H) if tok is None else out


def fp8_e4m3_encode(values: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_fp8_e4m3_encode(_p(v), _p(out), v.size)
    return out


def quantize_e4m3_blocks(rows: np.ndarray, block: int = 128):
    """rows [..., H] uint16 (bf16 bits) -> (codes [..., H] u8, scales [..., H/block] f32)."""
    r = np.ascontiguousarray(rows, dtype=np.uint16)
    H = r.shape[-1]
    n = r.size // H
    codes = np.empty(r.shape, np.uint8)
    scales = np.empty(r.shape[:-1] + (H // block,), np.float32)
    _check(lib().oracle_quantize_e4m3_blocks(_p(r), n, H, block, _p(codes), _p(scales)),
           "oracle_quantize_e4m3_blocks")
    return codes, scales


def lb_prefetch_weights(expert_weights, mapping, redundant_weights):
    """expert_weights [E, W] u16, mapping [N] i32 -> redundant_weights [N, W] u16 (updated copy)."""
    ew = np.ascontiguousarray(expert_weights, dtype=np.uint16)
    m = np.ascontiguousarray(mapping, dtype=np.int32)
    out = np.array(redundant_weights, dtype=np.uint16, copy=True, order="C")
    E, W = ew.shape
    _check(lib().oracle_lb_prefetch_weights(_p(ew), E, W, _p(m), m.size, _p(out)),
           "oracle_lb_prefetch_weights")
    return out


def lb_reduce_grads(redundant_grads, mapping, expert_grads, fp32: bool = False):
    """redundant_grads [N, W] u16, mapping [N] i32, expert_grads [E, W] u16 -> new expert_grads.
    fp32=False: the exact sum (fp64); fp32=True: the fixed-order definition (binary32
    additions from the original gradient over ascending replica index)."""
    rg = np.ascontiguousarray(redundant_grads, dtype=np.uint16)
    m = np.ascontiguousarray(mapping, dtype=np.int32)
    out = np.array(expert_grads, dtype=np.uint16, copy=True, order="C")
    E, W = out.shape
    fn = lib().oracle_lb_reduce_grads_fp32 if fp32 else lib().oracle_lb_reduce_grads
    _check(fn(_p(rg), _p(m), m.size, _p(out), E, W),
           "oracle_lb_reduce_grads" + ("_fp32" if fp32 else ""))
    return out
