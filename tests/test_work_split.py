"""The projection kernels' work decomposition, checked on the CPU.

tests/cpp/work_split_check.cu includes the very planning and walking
functions the persistent prefill and decode projections use (host/device
code) and walks them for hundreds of shapes: every (tile, k) unit processed
exactly once, split tiles' contributors and partial slots consistent with
what the last-arriving CTA reads back.  nvcc builds it for the host; no GPU
is needed to run it."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


def test_work_split_walks_cover_every_unit_once():
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    src = os.path.join(ROOT, "tests", "cpp", "work_split_check.cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "work_split_check")
        r = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                            "-I", os.path.join(ROOT, "include"), src, "-o", exe],
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-4000:]
        out = subprocess.run([exe], capture_output=True, text=True, timeout=600)
        assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout[-2000:] + out.stderr[-2000:]
