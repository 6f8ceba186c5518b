"""The bounds-checked build (libsaga_debug.so, compiled with SAGA_DEBUG) runs
the tiny workload and the edge shapes clean.  In that build every position,
count and slot a kernel takes from another kernel's output is checked before
use; one out of range sets a sticky bit that saga_workspace_error reports as
SAGA_ERR_BOUNDS (the access is skipped, no trap).  The parity tests below
assert a clean flag after every call, so a run that passes here had no
out-of-range index anywhere.  They run in a child process that loads the
debug library (SAGA_LIBRARY), which also checks it was the one loaded."""
import os
import subprocess
import sys

import pytest
import torch

from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200 import build as saga_build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELECTED = [
    "tests/test_gpu_parity.py::test_tiny_workload_32_steps",
    "tests/test_gpu_parity.py::test_short_and_ragged_caches",
    "tests/test_gpu_parity.py::test_stale_threshold_above_every_logit_keeps_the_maxima",
    "tests/test_gpu_parity.py::test_zero_query_and_unit_values",
    "tests/test_gpu_parity.py::test_N_at_least_l_equals_dense",
    "tests/test_gpu_one_row.py",
    "tests/test_gpu_refresh_step.py",
    "tests/test_gpu_growth.py",
]


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_debug_build_runs_the_edge_shapes_clean():
    if not os.path.exists(_lib.DEBUG_LIBRARY):
        saga_build.build(debug=True)
    env = dict(os.environ, SAGA_LIBRARY=_lib.DEBUG_LIBRARY)
    probe = ("from sparse_decode_attention_saga_b200 import _lib; _lib.load(); "
             "import os; print(os.path.realpath(_lib.LIBRARY))")
    r = subprocess.run([sys.executable, "-c", probe], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().endswith("libsaga_debug.so"), r.stdout
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider"]
                       + SELECTED, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert " passed" in r.stdout
