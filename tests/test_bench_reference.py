"""The benchmark's reference arm (the CPU oracle, timed) on the host: its one JSON
line carries the contract's keys; a non-zero rank exits without work."""
import contextlib
import io
import json
import os

import pytest


@pytest.fixture(scope="module")
def oracle_built():
    from oracle import build
    build.build()


def _run(argv, env=None):
    import bench
    old = {k: os.environ.get(k) for k in (env or {})}
    os.environ.update(env or {})
    buf = io.StringIO()
    try:
        with contextlib.redirect_stdout(buf):
            rc = bench.main(argv)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    return rc, buf.getvalue()


def test_reference_line(oracle_built):
    rc, out = _run(["--impl", "reference", "--steps", "2", "--warmup", "3", "--cpu-sample-tokens", "8"])
    assert rc == 0
    lines = [l for l in out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("dsv3")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"] and "sample" in cb
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_other_ranks_do_nothing(oracle_built):
    rc, out = _run(["--impl", "reference", "--steps", "1"], env={"RANK": "1", "WORLD_SIZE": "2"})
    assert rc == 0 and out.strip() == ""
