"""The measurement programs under tests/probes compile for sm_100a (CPU: nvcc
only, nothing runs).  profiles/ cites their output; this keeps them buildable."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROBES = os.path.join(ROOT, "tests", "probes")


@pytest.mark.parametrize("name", sorted(f for f in os.listdir(PROBES) if f.endswith(".cu")))
def test_probe_compiles(name, tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    out = tmp_path / name.replace(".cu", "")
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-I", os.path.join(ROOT, "entropy_adaptive_radius_b200", "csrc"),
                        "-o", str(out), os.path.join(PROBES, name), "-lcuda"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    assert out.exists()
