"""The small parity cases of the two persistent decode kernels, run against the TERN_DEBUG build
(libtern_debug.so): every shared- and global-memory index the kernels compute is checked before
its access, and a failed check is reported by tern_device_status instead of faulting. Each case
runs in a child pytest process with TERN_LIBRARY=debug (the library a process loads is fixed at
import) and TERN_CHECK_DEVICE_STATUS=1 (the autouse fixture of conftest.py then requires a clean
device status after every test)."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_debug(args):
    lib = os.path.join(ROOT, "ternary_weight_only_tern_b200", "libtern_debug.so")
    if not os.path.exists(lib):
        from ternary_weight_only_tern_b200 import build
        build.build(debug=True)
    env = dict(os.environ, TERN_LIBRARY="debug", TERN_CHECK_DEVICE_STATUS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider"] + args,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    return r.stdout


def test_the_debug_build_is_loaded_in_the_child():
    out = run_debug(["-k", "identify", os.path.join("tests", "test_abi.py")])
    assert "passed" in out


def test_one_token_kernel_small_cases_under_bounds_checks():
    run_debug([os.path.join("tests", "test_decode1_gpu.py"), "-k",
               "shapes_and_residual_fractions or exact_case or zero_plane or offsets or group_boundaries"])


def test_multi_token_kernel_small_cases_under_bounds_checks():
    run_debug([os.path.join("tests", "test_decodem_gpu.py"), "-k",
               "exact_case or zero_plane or group_boundaries or (shapes and 512-) or many_segments"])
