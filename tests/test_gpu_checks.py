"""The bounds-checking debug build (libsgqa_checks.so, built with -DSGQA_CHECKS).

Its kernels test every index and coordinate they compute from data (selections, union lists,
row permutations, reverse indices, cache positions) against the buffer it addresses; a failed
test records SGQA_ERR_DEVICE_CHECK and skips the access. These tests run the layer with it loaded
(in child processes, SGQA_LIBRARY=checks) and require (1) that no check fires on the parity
workloads, whose status assertions would catch SGQA_ERR_DEVICE_CHECK, and (2) that its results
equal the normal build's bit for bit, so the checks change nothing but the detection."""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _env(checks: bool):
    env = dict(os.environ)
    env.pop("SGQA_LIBRARY", None)
    if checks:
        env["SGQA_LIBRARY"] = "checks"
    return env


def test_checks_library_is_built():
    from block_sparse_long_kbar_b200 import build as b
    assert os.path.exists(b.build(variant="checks"))


def test_parity_suite_under_bounds_checks():
    cmd = [sys.executable, "-m", "pytest", "tests/test_gpu_parity.py", "tests/test_gpu_fp8.py", "tests/test_gpu_swa.py",
           "tests/test_gpu_backward.py", "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider",
           "-k", "not full_size and not largest_budget and not 1m"]
    r = subprocess.run(cmd, cwd=ROOT, env=_env(True), capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_checks_build_matches_normal_build_bitwise(tmp_path):
    paths = {}
    for checks in (False, True):
        p = str(tmp_path / f"res_{int(checks)}.npz")
        r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_layer_runner.py"), p], cwd=ROOT,
                           env=_env(checks), capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
        paths[checks] = p
    a, b = np.load(paths[False]), np.load(paths[True])
    assert str(a["library"]) == "libsgqa.so" and str(b["library"]) == "libsgqa_checks.so"
    for k in a.files:
        if k == "library":
            continue
        if "status" in k:
            assert int(a[k]) == 0 and int(b[k]) == 0, (k, int(a[k]), int(b[k]))
        else:
            assert np.array_equal(a[k], b[k]), k
