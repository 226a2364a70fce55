"""The bounds-checked debug build (libkvq_checked.so, -DKVQ_BOUNDS_CHECK).

Its kernels compare every checked cache, partial and window access with the
array's extent and count the ones out of bounds.  On the same small appends,
selections and decodes (plain, with bf16 token windows, and with
bucket-relative RoPE, a dual pair and windows together) it must give the
regular library's bytes and outputs exactly, with no access out of bounds;
the regular library reports that it has no checks (UINT32_MAX).
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def run(library):
    env = dict(os.environ)
    env["KVQ_LIBRARY"] = library
    r = subprocess.run([sys.executable, os.path.join(HERE, "bounds_worker.py")], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_checked_build_matches_the_regular_library_with_no_access_out_of_bounds():
    checked = run("checked")
    regular = run("regular")
    assert checked["violations"] == 0
    assert regular["violations"] == 0xFFFFFFFF
    assert checked["digest"] == regular["digest"]
