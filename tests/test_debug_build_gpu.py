"""The bounds-checked build (libbkv_debug.so, every data-dependent index in
the kernels guarded by BKV_CHECK) against the float64 oracle: a cross-section
of the parity cases runs on it, in a fresh process with BKV_LIBRARY=debug, so
that every kernel's checks are exercised and none fires (a fired check turns
the device status, which every parity case asserts to be clean, into
BKV_ERR_DEVICE_ASSERT)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = [
    "test_parity_gpu.py::test_score_select_compact",
    "test_parity_gpu.py::test_select_topk_exact",
    "test_parity_gpu.py::test_update_beacons",
    "test_parity_gpu.py::test_compress_step_small",
    "test_parity_gpu.py::test_compress_step_in_place",
    "test_parity_gpu.py::test_compress_step_query_ring",
]


def test_parity_on_the_debug_build():
    lib = os.path.join(ROOT, "kv_cache_compression_bkv_b200", "libbkv_debug.so")
    if not os.path.exists(lib):
        pytest.skip("libbkv_debug.so is not built")
    env = dict(os.environ, BKV_LIBRARY="debug")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           *[os.path.join(ROOT, "tests", c) for c in CASES]]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
    # the debug library is the one those tests loaded
    probe = subprocess.run([sys.executable, "-c",
                            "from kv_cache_compression_bkv_b200 import bkv; print(bkv.LIB_PATH)"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.stdout.strip().endswith("libbkv_debug.so"), probe.stdout + probe.stderr
