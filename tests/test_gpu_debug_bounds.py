"""The HSTU_DEBUG_BOUNDS build: every data-derived global index, TMA row
coordinate and workspace slot of the kernels passes a device-side check that
records a status bit instead of trapping.  The small-shape parity tests
(odd lengths 0, 1, 2, 127, 129, the fp32 tiny configuration, ragged
micro-batches) run against that build in a child process: they must pass
against the oracle with the device status clean (each of them checks the
status word after its calls)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELECTION = [
    "tests/test_gpu_forward.py::test_tiny_fp32_workload",
    "tests/test_gpu_forward.py::test_bf16_small",
    "tests/test_gpu_forward.py::test_fp32_small",
    "tests/test_gpu_forward.py::test_degenerate_shapes",
    "tests/test_gpu_forward.py::test_many_short_sequences",
    "tests/test_gpu_backward.py::test_bf16_backward_small",
    "tests/test_gpu_cand.py::test_small",
    "tests/test_gpu_proj.py::test_uvqk_small",
    "tests/test_gpu_proj.py::test_out_small",
]


def test_parity_with_device_index_checks():
    sys.path.insert(0, ROOT)
    from pointwise_attention_b200 import build
    lib = build.build(debug_bounds=True)
    assert lib.endswith("libhstu_debug.so")
    env = dict(os.environ, HSTU_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider"] +
                       SELECTION, cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=1200)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in tail and "failed" not in tail, tail
