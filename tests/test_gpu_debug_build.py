"""The bounds-checking debug build (-DSVDQ_DEBUG) on small odd shapes.

In libsvdq_debug.so every plain global or shared-memory access of the kernels checks its
index first and, out of bounds, skips the access and records site 201 (global) or 202
(shared) in the device error word.  Each library runs in a child process of its own
(tests/debug_child.py): the layer must finish every format and shape with a clean device
error word under the debug build, and give the release build's output bit for bit.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "bit_w4a4_quantized_group_b200", "_lib")


def _run(lib, out):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_child.py"), lib, out],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return dict(np.load(out))


@pytest.mark.gpu
def test_debug_build_is_clean_and_matches_release(tmp_path):
    from bit_w4a4_quantized_group_b200 import build as BUILD
    debug_lib = BUILD.build(debug=True)        # up to date in the tree; builds it otherwise
    release_lib = BUILD.build()
    dbg = _run(debug_lib, str(tmp_path / "debug.npz"))
    rel = _run(release_lib, str(tmp_path / "release.npz"))
    assert list(dbg["device_error"]) == [0, 0], dbg["device_error"]
    assert list(rel["device_error"]) == [0, 0], rel["device_error"]
    keys = sorted(k for k in rel if k != "device_error")
    assert keys == sorted(k for k in dbg if k != "device_error")
    assert len(keys) == 16
    for k in keys:
        assert np.array_equal(dbg[k], rel[k]), k
