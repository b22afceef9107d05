"""Host check of the sequence-parallel row map of the GEMM producers (seq_row and its
incremental SeqCursor, from the library's own header), compiled with nvcc for the host and run
on the CPU: the map is the shard-major layout [p][b][s/p] of token (b, pos), a bijection, and
the cursor returns it for every 64-token step of repeated sweeps."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_seq_row_and_cursor_on_host():
    src = os.path.join(HERE, "host", "seq_cursor_check.cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "seq_cursor_check")
        r = subprocess.run([_nvcc(), "-std=c++17", "-O1", "-o", exe, src],
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
