"""The debug build (libcsa2_debug.so: NVTX ranges per C-ABI call and
device-side bounds checks on every position and page, -DCSA2_NVTX
-DCSA2_DEBUG_BOUNDS) gives the same parity results: whole stacks of every
workload against the oracle, and the out-of-range cases flagged in the status
word, never trapped.  The tests run in a child process that loads the debug
library (CSA2_LIBRARY=debug)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = ["tests/test_gpu_stack.py::test_stack_small",
         "tests/test_gpu_attn.py::test_out_of_range_topk_flags_status",
         "tests/test_gpu_index.py::test_out_of_range_pool_entry_flags_status",
         "tests/test_gpu_quant.py::test_out_of_range_append_flags_status",
         "tests/test_gpu_export.py::test_export_outside_the_cache_is_zero_and_flagged",
         "tests/test_gpu_cp.py::test_cp_empty_parts_and_bad_topk_entries",
         "tests/test_gpu_debug_build.py::test_loaded_library_is_the_debug_build"]


def test_loaded_library_is_the_debug_build():
    if os.environ.get("CSA2_LIBRARY") != "debug":
        pytest.skip("runs inside the debug-build child process")
    import fp4_sparse_attention_csa2_b200 as csa2
    csa2.lib()
    assert os.path.basename(csa2.LIB_PATH) == "libcsa2_debug.so"
    with open("/proc/self/maps") as f:
        assert "libcsa2_debug.so" in f.read()


def test_parity_under_the_debug_build():
    from fp4_sparse_attention_csa2_b200 import build
    build.build(debug=True)
    env = dict(os.environ, CSA2_LIBRARY="debug")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", *CASES], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
