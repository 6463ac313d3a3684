"""The checking build (libcowa_debug.so, COWA_DEBUG=1: the kernels check
tile, row and workspace indices against their extents and report a failed
check as COWA_ERR_DEVICE) runs the small ragged parity cases of every kernel
in a process of its own, with no check failing and the results matching the
oracle.  The release build runs the same cases for comparison."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("debug", [True, False])
def test_checked_cases(debug):
    from structured_sparse_attention_block_b200 import build
    lib = build.build(debug=debug)
    env = dict(os.environ)
    env["COWA_DEBUG"] = "1" if debug else "0"
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_cases.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert ("checked ok %s" % lib) in r.stdout
