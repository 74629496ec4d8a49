"""Programmatic dependent launch (opt-in with SDV_PDL=1): every kernel waits on the previous
grid before its first global access, so results must not change.  Reruns a cross-section of
the parity tests in a child process with the launches made programmatic."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELECTION = [
    "tests/test_gpu_attention.py::test_verify_bf16_small",
    "tests/test_gpu_attention.py::test_verify_window",
    "tests/test_gpu_attention.py::test_verify_split_across_ctas",
    "tests/test_gpu_attention.py::test_draft_xattn",
    "tests/test_gpu_lm_head.py::test_clustered_small",
    "tests/test_gpu_lm_head.py::test_drafter_clustered_config",
    "tests/test_gpu_accept.py::test_full_vocab_sampling",
    "tests/test_gpu_accept.py::test_plain_draw_dense_rows_twice_on_one_workspace",
    "tests/test_gpu_commit.py",
]


def test_parity_with_programmatic_launches():
    env = dict(os.environ, SDV_PDL="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", *SELECTION],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
