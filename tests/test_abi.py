"""CPU checks of the C ABI: the library builds, loads and exports every symbol the
header declares; host-side validation rejects bad shapes before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from combine_ep_get_11_b200 import build
    build.build()
    import combine_ep_get_11_b200 as ep
    return ep.load()


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("ep_create", "ep_destroy", "ep_get_dispatch_layout", "ep_dispatch",
                     "ep_dispatch_cached", "ep_combine", "ep_ll_dispatch", "ep_ll_combine",
                     "ep_sync_status", "ep_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    for code, name in [(0, b"EP_OK"), (1, b"EP_ERR_INVALID_ARG"), (2, b"EP_ERR_ALIGNMENT"),
                       (3, b"EP_ERR_CAPACITY"), (4, b"EP_ERR_BAD_TOPK"),
                       (5, b"EP_ERR_HANDLE_MISMATCH"), (6, b"EP_ERR_TIMEOUT"), (7, b"EP_ERR_CUDA"),
                       (8, b"EP_ERR_UNIMPLEMENTED")]:
        assert lib.ep_status_string(code) == name


@pytest.mark.parametrize("cfg,code", [
    ((0, 8, 64, 256, 2, 10, 0), 1),        # no ranks
    ((33, 33, 64, 256, 2, 10, 0), 1),      # more ranks than a warp
    ((4, 10, 64, 256, 2, 10, 0), 1),       # experts not divisible by ranks
    ((2, 8, 64, 250, 2, 10, 0), 2),        # rows not whole 16-byte vectors
    ((2, 8, 64, 256, 0, 10, 0), 1),        # top-0
    ((2, 8, 64, 256, 33, 10, 0), 1),       # top-k wider than a warp
    ((2, 8, 64, 256, 2, 0, 0), 1),         # no channels
    ((2, 8, 64, 256, 2, 10, 32), 1),       # Tmax below T
    ((2, 8, -1, 256, 2, 10, 0), 1),        # negative tokens
])
def test_bad_config_is_rejected_on_the_host(lib, cfg, code):
    import combine_ep_get_11_b200 as ep
    c = ep.ep_config(*cfg)
    out = ctypes.c_void_p()
    assert lib.ep_create(ctypes.byref(c), ctypes.byref(out)) == code
    assert out.value is None


def test_null_arguments(lib):
    assert lib.ep_create(None, None) == 1
    assert lib.ep_destroy(None) == 1
    assert lib.ep_sync_status(None, None) == 1
    assert lib.ep_dispatch(None, *([None] * 10), 0, None, None, None) == 1


def test_no_kernels_launched_on_cpu(lib):
    assert lib.ep_kernel_launch_count() == 0


@pytest.mark.parametrize("shards,shard", [(3, 0), (0, 0), (2, 2), (2, -1), (33, 0)])
def test_bad_shard_split_is_rejected_on_the_host(lib, shards, shard):
    import combine_ep_get_11_b200 as ep
    c = ep.ep_config(8, 64, 16, 256, 2, 10, 0)
    out = ctypes.c_void_p()
    assert lib.ep_create_sharded(ctypes.byref(c), shards, shard, ctypes.byref(out)) == 1
    assert out.value is None


def test_sharded_null_arguments(lib):
    assert lib.ep_sharded_handle(None, *([None] * 9)) == 1
    assert lib.ep_sharded_dispatch(None, None, None, None, None, None, 1, None, None, None, None, 0,
                                   None, None) == 1
    assert lib.ep_sharded_combine(None, 1, None, None, 0, None, None, None, None, None, None, None, None) == 1
    assert lib.ep_shared_alloc(0, None, None) == 1
    assert lib.ep_ipc_open(None, None) == 1


def test_check_and_test_support_null_arguments(lib):
    assert lib.ep_check_handle(None, None, None, None, None) == 1
    assert lib.ep_test_offset_tickets(None, 1) == 1
    assert lib.ep_get_num_recv(None, None, None, None, None, None) == 1
