"""The debug build (device-side bounds checks, see video_dit_local_b200/build.py)
and guard bytes around every output.

tests/_entry_point_canaries.py runs every data entry point on small grids
with canary bytes around each output and workspace; it runs once with the
default library and once with the debug build, each in its own process.  In
both, every call must leave the status word at VATTN_OK (the debug build
would report VATTN_ERR_DEVICE_BOUNDS for any out-of-range row, tile or TMA
coordinate it computed) and every canary intact; the two builds' outputs must
be bit-identical (the checks add branches, not arithmetic), except dg, whose
per-block partials are summed with atomics in a varying order.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRIPT = os.path.join(ROOT, "tests", "_entry_point_canaries.py")

pytestmark = pytest.mark.gpu


def _run(tmp_path, debug: bool):
    env = dict(os.environ)
    env.pop("VATTN_DEBUG_BUILD", None)
    if debug:
        env["VATTN_DEBUG_BUILD"] = "1"
    out = tmp_path / ("debug.npz" if debug else "default.npz")
    r = subprocess.run([sys.executable, SCRIPT, str(out)], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, f"{'debug' if debug else 'default'} build: {r.stdout[-2000:]} {r.stderr[-4000:]}"
    return np.load(out)


def test_debug_build_checks_pass_and_match_the_default_build(tmp_path):
    import importlib.util
    spec = importlib.util.spec_from_file_location("_vattn_build", os.path.join(ROOT, "video_dit_local_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build(debug=True)          # no-op when the in-tree debug library is current
    ref = _run(tmp_path, debug=False)
    dbg = _run(tmp_path, debug=True)
    assert sorted(ref.files) == sorted(dbg.files)
    for name in ref.files:
        if name == "dg":  # sums per-block partials with atomics: the order of the adds varies
            np.testing.assert_allclose(ref[name], dbg[name], rtol=1e-5, atol=1e-6)
        else:
            assert np.array_equal(ref[name], dbg[name]), name
