"""The debug build (libkda_debug.so, kernels with index checks) on the GPU: a selection of
the parity tests runs in a child process that loads it, and every one must pass with no
check firing (a fired check fails the tests through kda_device_status)."""
import os
import subprocess
import sys

import pytest

from chunked_linear_attention_chunk_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_tests_pass_on_the_debug_build():
    build.build(debug_checks=True)
    env = dict(os.environ, KDA_DEBUG_CHECKS="1")
    which = subprocess.run([sys.executable, "-c", "import chunked_linear_attention_chunk_b200 as k; print(k.LIB_PATH)"],
                           cwd=ROOT, env=env, capture_output=True, text=True, check=True).stdout.strip()
    assert which.endswith("libkda_debug.so"), which
    sel = ["tests/test_chunk_gpu.py::test_bf16_several_chunks_ragged_tail",
           "tests/test_chunk_gpu.py::test_bf16_edge_lengths",
           "tests/test_chunk_gpu.py::test_prep_then_scan_equals_one_call_bitwise",
           "tests/test_varlen_gpu.py", "tests/test_sp_gpu.py::test_three_segments_on_one_gpu_match_one_run",
           "tests/test_logsigmoid_gpu.py::test_logsig_edge_lengths",
           "tests/test_bwd_gpu.py::test_bwd_matches_oracle", "tests/test_bwd_gpu.py::test_bwd_varlen_matches_oracle"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", *sel], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
