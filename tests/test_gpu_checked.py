"""The bounds-checked build (libmx_checked.so, -DMX_CHECKED): every global store of every
kernel is checked against the output extents its launcher registered, computed on the
host from the shapes.  Run in a subprocess (one library per process): every case must
match the oracle with no store refused; then, with the registered extent of the last
output shortened by a test hook, the kernel's stores beyond it must be refused and
reported (watchdog code 64) -- a check that the checking works, made without any
out-of-bounds access (the refused stores are inside the real buffer)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(cases, shrink=None):
    from microscaling_precision_number_b200 import build
    lib = build.build(checked=True)
    env = dict(os.environ, MX_LIB_PATH=lib)
    if shrink is not None:
        env["MX_CHECKED_SHRINK"] = str(shrink)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_run.py")] + cases, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_checked_build_every_case_in_bounds():
    res = run([])
    for name, r in res.items():
        assert r["match"], name
        assert r["watchdog"] == 0, (name, r)


def test_checked_build_refuses_stores_beyond_a_registered_extent():
    # the last registered range of a row-wise quantisation is its tcgen05 scale array: cut
    # 16 bytes off it, and the scale stores that land there are refused and reported
    res = run(["rows_e4m3_37x96"], shrink=16)
    assert res["rows_e4m3_37x96"]["watchdog"] == 64
