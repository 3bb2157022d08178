"""The GEMM's work split is chosen per call (global stream-K, or cluster
split-K with 2, 4 or 8 CTAs per tile), INT4 weights are widened ahead of
the GEMM for large token counts, and kernels are chained with
programmatic dependent launch.  The environment switches read once per
process force each variant, so every one of them is checked against the
oracle here: the exact INT32 accumulators of the split-K test and the
ragged-shape sweep, each in a fresh process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MODES = [
    {"QLIN_NO_CLUSTER": "1"},   # global stream-K for every split tile
    {"QLIN_CLUSTER_CS": "2"},
    {"QLIN_CLUSTER_CS": "4"},
    {"QLIN_CLUSTER_CS": "8"},
    {"QLIN_NO_PDL": "1"},       # plain stream-ordered launches
    {"QLIN_WIDEN_MIN_M": "129"},  # INT4 weights widened once, INT8 kernel, from 129 tokens
    {"QLIN_WIDEN_MIN_M": "0"},    # INT4 converters in the GEMM for every token count
]


@pytest.mark.parametrize("env", MODES, ids=lambda e: ",".join(f"{k}={v}" for k, v in e.items()))
def test_forced_split_mode(env):
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
           "tests/test_gpu_fullsize.py::test_split_k_accumulators_exact",
           "tests/test_gpu_parity.py::test_shapes"]
    r = subprocess.run(cmd, cwd=ROOT, env={**os.environ, **env}, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-4000:], r.stderr[-2000:])
