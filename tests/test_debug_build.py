"""The debug build (libtbq4_debug.so, compiled with -DTBQ4_DEBUG) switches on
the kernels' bounds checks: every global access a kernel derives from
lengths, positions, page ids or its split plan is checked against its
buffer's extent, and a failed check is reported as TBQ4_ERR_BOUNDS.

This runs every entry point on the same seeded inputs twice, each in a fresh
process: once on the release library, once on the debug library
(TBQ4_DEBUG=1).  No check may fire (status 0), and every cache byte and
every output must be the same bit for bit: the checks only observe.  The
outputs themselves are compared with the oracle by the other test files.
"""
import importlib.util
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _build_debug():
    spec = importlib.util.spec_from_file_location(
        "tbq4_build", os.path.join(ROOT, "long_context_attention_tbq4_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    return build.build(debug=True)


def _run(tmp_path, debug):
    out = tmp_path / ("debug.npz" if debug else "release.npz")
    env = dict(os.environ, TBQ4_DEBUG="1" if debug else "0")
    subprocess.run([sys.executable, os.path.join(HERE, "debug_build_cases.py"), str(out)],
                   env=env, check=True, timeout=900)
    return np.load(out)


def test_debug_build_matches_release_bit_for_bit(tmp_path):
    _build_debug()
    rel = _run(tmp_path, debug=False)
    dbg = _run(tmp_path, debug=True)
    assert int(rel["debug"]) == 0 and int(dbg["debug"]) == 1
    assert list(rel["mapped"]) == ["libtbq4.so"], rel["mapped"]
    assert list(dbg["mapped"]) == ["libtbq4_debug.so"], dbg["mapped"]
    assert int(rel["status"]) == 0
    assert int(dbg["status"]) == 0, "a bounds check of the debug build fired"
    keys = [k for k in rel.files if k not in ("debug", "lib", "mapped")]
    assert len(keys) >= 12
    for k in keys:
        np.testing.assert_array_equal(rel[k], dbg[k], err_msg=k)
