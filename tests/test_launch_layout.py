"""Host-side invariants of the launch geometry: the decode kernel's cluster
size and shared-memory layout for every supported shape, and the other
kernels' shared-memory sizes against the opt-in limit. tests/host/layout_check.cu
is compiled against the library's own headers and run on the CPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(nvcc() is None, reason="nvcc not found")
def test_launch_layout_invariants(tmp_path):
    exe = tmp_path / "layout_check"
    subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "--expt-relaxed-constexpr",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "rank_key_top_b200", "csrc"),
                    os.path.join(ROOT, "tests", "host", "layout_check.cu"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout
    assert "layout ok" in res.stdout
    # the shapes the tests and the benchmark use are all supported
    for line in res.stdout.splitlines():
        if line.startswith("unsupported from L="):
            assert int(line.split("=")[1].split(":")[0]) > 16384, line
