"""The debug build's device-side index checks (libssd_debug.so, -DSSD_DEBUG_BOUNDS).

Each build runs in a subprocess of its own (tests/bounds_case.py).  With the full extents the
checked build gives bit-identical outputs and no error.  With the test hook allowing half of
each buffer's extent, the call trips the checks on valid buffers, so every access stays inside
its allocation: the device error word holds SSD_ERR_DEVICE_BOUNDS, the skipped stores leave
the second half of the rows of y and of the heads of h_final as they were (NaN), and what the
call could still compute from unskipped inputs (the first half of the rows, the heads whose dt
and prefix sums were written) matches the normal build bit for bit."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SSD_ERR_DEVICE_BOUNDS = 6


def _run(tmp_path, lib, denom, norm_groups):
    out = str(tmp_path / f"out_{os.path.basename(lib)}_{denom}_{norm_groups}.npz")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bounds_case.py"), lib, str(denom),
                        str(norm_groups), out], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return dict(np.load(out))


@pytest.mark.parametrize("norm_groups", [0, 2])
def test_index_checks_of_the_debug_build(cuda_lib, tmp_path, norm_groups):
    from mamba_ssd_scan_02_b200 import ssd
    if not os.path.exists(ssd.DEBUG_LIB_PATH):  # normally built beside libssd.so by build()
        from mamba_ssd_scan_02_b200 import build as _b
        _b.build(debug_bounds=True)
    ref = _run(tmp_path, ssd.LIB_PATH, 1, norm_groups)
    assert ref["debug_build"] == 0 and ref["status"] == 0
    full = _run(tmp_path, ssd.DEBUG_LIB_PATH, 1, norm_groups)
    assert full["debug_build"] == 1 and full["status"] == 0
    assert np.array_equal(full["y"], ref["y"], equal_nan=True)
    assert np.array_equal(full["h_final"], ref["h_final"], equal_nan=True)
    half = _run(tmp_path, ssd.DEBUG_LIB_PATH, 2, norm_groups)
    assert half["status"] == SSD_ERR_DEVICE_BOUNDS
    rows, heads = ref["y"].shape[1] // 2, ref["h_final"].shape[1] // 2
    assert np.isnan(half["y"][0, rows:]).all() and np.isnan(half["h_final"][0, heads:]).all()
    c = heads * 64
    assert np.array_equal(half["y"][0, :rows, :c], ref["y"][0, :rows, :c])
    assert np.array_equal(half["h_final"][0, :heads], ref["h_final"][0, :heads])
