"""The boundary is a C ABI: a plain C program compiled with gcc against
include/waveprune.h and linked to libwaveprune.so calls it (host-side calls
only) and gets the same results as the Python binding."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import rope_period_truncated_b200 as wp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_caller(tmp_path):
    lib = wp.library_path()
    assert os.path.exists(lib), "build the library first"
    exe = tmp_path / "abi_smoke"
    subprocess.check_call(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi", "abi_smoke.c"), "-o", str(exe),
                           "-L", os.path.dirname(lib), "-lwaveprune", "-Wl,-rpath," + os.path.dirname(lib)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    grp = [int(x) for x in out[0].split()]
    _, wg = wp.wp_cutoffs(128, 1e6, wp.ROPE_HALF_SPLIT)
    assert grp == [int(x) for x in wg]
    counts = np.array([int(x) for x in out[1].split()]).reshape(8, 3)
    _, ref = wp.wp_schedule(4096, 128, 128, wg, want_map=False)
    assert np.array_equal(counts, np.asarray(ref).reshape(8, 3))
    code, text = out[2].split(" ", 1)
    assert int(code) == wp.WP_ERR_ARG and text == wp.wp_status_str(wp.WP_ERR_ARG)
