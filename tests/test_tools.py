"""CPU checks of the developer tools that ship with the package."""

import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_trace_tool_command_line():
    """The pipeline trace tool parses its arguments and names every workload
    (it builds and runs only with a GPU; --help exits first)."""
    r = subprocess.run([sys.executable, "-m", "ulysses_sequence_attention_sp_b200.trace", "--help"],
                       capture_output=True, text=True, cwd=ROOT, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "--workload" in r.stdout
    for name in ("vit", "video", "chunked", "hybrid"):
        assert name in r.stdout
