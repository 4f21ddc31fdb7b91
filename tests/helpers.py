"""Shared test utilities: bf16 bit views, the combine tolerance, GPU runners."""
from __future__ import annotations

import os

import numpy as np
import torch

import synth


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_bf16_tensor(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_abs(a: np.ndarray) -> np.ndarray:
    return (a & np.uint16(0x7FFF)).astype(np.uint16)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (8 significant bits; subnormals step 2^-133)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def combine_tolerance(ref: np.ndarray, got: np.ndarray, abs_sum: np.ndarray | None, n_terms: int):
    """Allowed |got - ref| for an fp32 accumulation of n_terms rounded to bf16, against the
    fp64-accumulated oracle value ref (also rounded to bf16):
      half a bf16 ulp of each rounding + the fp32 accumulation bound n*2^-24*sum|terms|.
    With no cancellation this is the 1 bf16 ulp bar."""
    r, g = bf16_to_f64(ref), bf16_to_f64(got)
    tol = 0.5 * bf16_ulp(r) + 0.5 * bf16_ulp(g)
    if abs_sum is not None:
        tol = tol + 1.01 * n_terms * 2.0 ** -24 * bf16_to_f64(abs_sum)
    return np.abs(g - r), tol


def assert_combine_close(got: np.ndarray, ref: np.ndarray, abs_sum=None, n_terms=8, what="",
                         return_ratio=False):
    diff, tol = combine_tolerance(ref, got, abs_sum, n_terms)
    bad = diff > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; first at {tuple(i)}: "
            f"got {bf16_to_f64(got)[tuple(i)]!r} ref {bf16_to_f64(ref)[tuple(i)]!r} tol {tol[tuple(i)]!r}")
    if return_ratio:
        return diff, tol
    ulps = diff / bf16_ulp(bf16_to_f64(ref))
    return float(ulps.max()) if ulps.size else 0.0, float(diff.mean()) if diff.size else 0.0


GOLDEN_FP32 = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fp32_order.txt")


def load_golden_fp32() -> dict:
    """The hand-worked fp32 summation-order cases (tests/golden/fp32_order.txt):
    key -> list of ints (hex bit patterns or decimals)."""
    vals = {}
    with open(GOLDEN_FP32) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [int(v, 16) if v.lower().startswith(("0x", "-0x")) else int(v) for v in rest]
    return vals


# (case, statistics) of every combine checked in this session; printed in the
# test summary by conftest.py
COMBINE_REPORT: list = []


def combine_stats(got: np.ndarray, exact: np.ndarray) -> dict:
    """Error of bf16 results against the exact sums rounded to bf16: max error in
    bf16 ulps (of the exact value), max relative error, mean absolute error."""
    g, r = bf16_to_f64(got), bf16_to_f64(exact)
    diff = np.abs(g - r)
    if diff.size == 0:
        return {"n": 0, "max_ulp": 0.0, "max_rel": 0.0, "mean_abs": 0.0}
    nz = r != 0
    rel = np.where(nz, diff / np.where(nz, np.abs(r), 1.0), np.where(diff > 0, np.inf, 0.0))
    return {"n": int(diff.size), "max_ulp": float((diff / bf16_ulp(r)).max()),
            "max_rel": float(rel.max()), "mean_abs": float(diff.mean())}


def check_combine(what: str, got: np.ndarray, fp32_ref: np.ndarray, exact: np.ndarray,
                  abs_sum=None, n_terms: int = 8, one_ulp: bool = False, cancelling: bool = False) -> dict:
    """A GPU combine result: bit-exact against the oracle's fixed-order fp32
    definition; against the exact sum either within one bf16 ulp (one_ulp: the
    accuracy bar for N(0,1) rows) or within the binary32 summation bound
    (abs_sum: a sum whose terms cancel can lose every bit of a small result, so
    only the bound applies).  The error statistics are recorded for the test
    summary: in ulps for ordinary rows, as a fraction of the bound for rows whose
    terms cancel (cancelling)."""
    np.testing.assert_array_equal(got, fp32_ref, err_msg=f"{what}: fixed-order fp32 definition")
    st = combine_stats(got, exact)
    st["differ"] = float(np.mean(got != exact)) if got.size else 0.0
    if one_ulp:
        assert st["max_ulp"] <= 1.0, f"{what}: {st['max_ulp']} ulp from the exact sum"
    if abs_sum is not None:
        diff, tol = assert_combine_close(got, exact, abs_sum, n_terms, what, return_ratio=True)
        st["bound_used"] = float((diff / tol).max()) if diff.size else 0.0
    st["cancelling"] = cancelling
    COMBINE_REPORT.append((what, st))
    return st


class Inputs:
    """Seeded inputs of one workload, on the host (numpy / CPU torch) and on the GPU."""

    def __init__(self, w: synth.Workload, device="cuda"):
        self.w = w
        self.topk = synth.topk_idx(w)
        self.weights = synth.topk_weights(w)
        self.x = synth.hidden_rows(w)
        self.x_u16 = u16(self.x)
        self.topk_d = torch.from_numpy(self.topk).to(device)
        self.weights_d = torch.from_numpy(self.weights).to(device)
        self.x_d = self.x.to(device)


def identity_combine_closed_form(fan: np.ndarray, x_u16: np.ndarray) -> np.ndarray:
    """Combine of identity experts, token by token: fan copies of x summed from +0.
    The sum is exact (fan * x fits in fp32), so it is bf16(fan * x) with one rounding --
    except for zeros: +0 plus any number of signed zeros is +0 under round-to-nearest."""
    xb = torch.from_numpy(np.ascontiguousarray(x_u16).view(np.int16)).view(torch.bfloat16)
    f = torch.from_numpy(np.ascontiguousarray(fan, dtype=np.float32))
    out = (f[..., None] * xb.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = out.copy()
    out[out == 0x8000] = 0
    return out
