import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library's Python binding (fails loudly if the build is missing)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test collected on a machine without CUDA")
    import combine_ep_get_11_b200 as ep
    ep.load()
    return ep


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Combine error statistics of the GPU tests (bit-exact against the oracle's
    fixed-order fp32 definition; these figures are against the exact sums)."""
    helpers = sys.modules.get("helpers")
    rows = getattr(helpers, "COMBINE_REPORT", None) if helpers is not None else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("combine error against the exact sum (results equal the fixed-order fp32 oracle bit for bit)")
    tr.write_line("N(0,1) rows: max error in bf16 ulps of the exact sum, max relative error, mean abs error; "
                  "cancelling rows: share of elements off the exact sum and the largest error as a "
                  "fraction of the binary32 summation bound")
    for what, st in rows:
        if st.get("cancelling"):
            tail = f"differ={st['differ']:<8.3g} max_err/bound={st['bound_used']:.3g}"
        else:
            tail = f"max_ulp={st['max_ulp']:<5.3g} max_rel={st['max_rel']:<9.3g} mean_abs={st['mean_abs']:.3e}"
        tr.write_line(f"{what:72s} n={st['n']:>9d}  {tail}")
