"""The bounds-checking build (-DUSP_BOUNDS_CHECK) against the layout, row,
ring, TMA-pack, guard-band and rank-local (multi-process) tests.

In that build every global offset the copy kernels and the attention
epilogues compute is checked against its buffer's extent; an out-of-range
one is skipped and its site recorded, and usp_device_status then reports it
(the tests assert it reports 0). The tests run in a child process that loads
the checked library through $USP_LIBRARY."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["tests/test_gpu_layout.py", "tests/test_gpu_rows.py", "tests/test_gpu_ring.py",
         "tests/test_gpu_pack_tma.py", "tests/test_gpu_guard_bands.py", "tests/test_gpu_dist.py",
         "tests/test_gpu_two_tile.py"]


def test_checked_build_passes_the_copy_and_attention_tests():
    from ulysses_sequence_attention_sp_b200 import build

    lib = build.build_checked()
    env = dict(os.environ, USP_LIBRARY=lib)
    res = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *FILES],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert res.returncode == 0, res.stdout[-4000:] + res.stderr[-2000:]
