"""The debug-bounds build (libosdn_debug.so, compiled with -DOSDN_DEBUG_BOUNDS: every computed
row or slot index of the kernels' global stores is checked against its buffer before the store)
on the GPU: on every entry point, both io dtypes, both head sizes, packed sequences with empty and
one-token members and the 1.3B-layer shape, it leaves the device status word OK (no check fired)
and gives the release build's outputs bit for bit (the checks change no arithmetic).  Each build
runs in a process of its own (tests/debug_bounds_run.py), since a process loads one library.
"""
import json
import os
import subprocess
import sys

import pytest

from delta_rule_recurrent_osdn_b200 import build as B

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(lib, out):
    env = dict(os.environ, OSDN_LIBRARY=lib)
    subprocess.run([sys.executable, "-m", "tests.debug_bounds_run", str(out)], cwd=ROOT, env=env,
                   check=True, timeout=900)
    with open(out) as f:
        return json.load(f)


def test_debug_bounds_build_matches_release(tmp_path):
    B.build()
    B.build(debug_bounds=True)
    rel = run(B.LIB, tmp_path / "release.json")
    dbg = run(B.DEBUG_LIB, tmp_path / "debug.json")
    assert rel.pop("library") == B.LIB and dbg.pop("library") == B.DEBUG_LIB
    assert rel.keys() == dbg.keys()
    for case in rel:
        assert rel[case]["status"] == 0, (case, "release", rel[case]["status"])
        assert dbg[case]["status"] == 0, (case, "debug-bounds", dbg[case]["status"])
        assert dbg[case]["outputs"] == rel[case]["outputs"], case
