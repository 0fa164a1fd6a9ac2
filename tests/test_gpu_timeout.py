"""Failure detection: a bounded device wait that runs out is reported, and the
context stays usable.

Every wait in the library's kernels is bounded; one that runs out records
PRISM_ERR_TIMEOUT in the workspace status word, the kernel drains its copies
and products, releases its tensor memory and returns. This test builds the
test variant of the library (dynamic_block_sparse_shape_b200.build
FAULT_INJECTION_FLAGS: waits give up after 50 ms, and a workspace word makes
the forward's copy producer skip one step's copies of one CTA) and runs it in a
child process that loads only that variant. The child sets the word, runs the
forward once normally, sets the word, runs it again (its score issuer then
waits for copies nobody issued), reads the status, clears the word and runs
the same forward once more in the same context.
The test asserts that the first call returned with PRISM_ERR_TIMEOUT in well
under the wait limit of the product build, and that the second call reports
PRISM_OK and matches the fp64 oracle within max-abs 2e-2 / mean-abs 2e-3.
"""
import json
import os
import subprocess
import sys

import pytest

from dynamic_block_sparse_shape_b200 import build as _build
from tests.gpu_util import ATOL_MAX, ATOL_MEAN, require_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_forward_wait_timeout_is_reported_and_the_context_recovers():
    require_gpu()
    lib = _build.build_variant("faultinj", _build.FAULT_INJECTION_FLAGS)
    env = dict(os.environ, PRISM_LIBRARY=lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "tests.timeout_child"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("REPORT ")]
    assert line, r.stdout[-2000:] + r.stderr[-2000:]
    rep = json.loads(line[-1][len("REPORT "):])
    print(rep)
    assert rep["library"] == lib
    assert rep["status"] == "PRISM_ERR_TIMEOUT"
    assert rep["faulted_call_s"] < 1.5  # a few 50 ms waits, not the product build's 2 s limit
    assert rep["status_after"] == "PRISM_OK"
    assert rep["o_max_abs"] <= ATOL_MAX and rep["o_mean_abs"] <= ATOL_MEAN
    assert rep["lse_max_abs"] <= ATOL_MAX
