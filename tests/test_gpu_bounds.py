"""The debug-bounds build (libowq_b200_bounds.so, -DOWQ_DEBUG_BOUNDS): device index checks on
every data-dependent access (the weak index list in each gather and scatter, the storage-stream
positions) that report OWQ_ERR_BOUNDS through owq_device_status instead of faulting.

The same seeded cases (quantise, storage pack / unpack, decode, prefill, both input-gradient
paths, both weak-gradient kernels) run once through each build, in separate processes
(tests/bounds_run.py); the outputs must agree bit for bit and the debug build must report no
failed check.  Then OWQ_INJECT_BOUNDS plants one out-of-range store index in the input
gradient's weak pass: the check must skip it and report OWQ_ERR_BOUNDS, and every other output
must be unchanged.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "weight_only_mixed_owq_b200")


def _run(variant, out, *extra):
    env = dict(os.environ, OWQ_LIB_VARIANT=variant)
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bounds_run.py"), out, *extra],
                          env=env, capture_output=True, text=True, timeout=600)
    assert proc.returncode == 0, proc.stdout[-2000:] + proc.stderr[-4000:]
    return np.load(out)


def test_debug_bounds_build_matches_and_reports(tmp_path):
    if not os.path.exists(os.path.join(PKG, "libowq_b200_bounds.so")):
        from weight_only_mixed_owq_b200 import build as b
        b.build(debug_bounds=True)
    ref = _run("", str(tmp_path / "default.npz"))
    dbg = _run("bounds", str(tmp_path / "bounds.npz"), "--inject")
    assert str(ref["version"]) == "0.1.0" and str(dbg["version"]).endswith("+debug-bounds")
    OWQ_OK, OWQ_ERR_BOUNDS = 0, 13
    compared = 0
    for key in ref.files:
        if key == "version":
            continue
        assert key in dbg.files, key
        if key.endswith("_status"):
            assert int(ref[key]) == OWQ_OK and int(dbg[key]) == OWQ_OK, (key, int(ref[key]), int(dbg[key]))
            continue
        a, b = ref[key], dbg[key]
        assert a.shape == b.shape and a.dtype == b.dtype, key
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f"{key}: the builds differ"
        compared += 1
    assert compared >= 20
    # the planted index: reported, skipped, nothing else touched
    assert int(dbg["inject_status"]) == OWQ_ERR_BOUNDS
    clean, planted = dbg["inject_clean"], dbg["inject_planted"]
    idx0 = int(dbg["c0_idx"][0])
    differ = np.argwhere(clean.view(np.uint16) != planted.view(np.uint16))
    assert all(tuple(p) == (0, idx0) for p in differ), differ[:5]
