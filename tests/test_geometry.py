"""The GEMV work split (host-side planning shared with the engine's setup),
checked on the CPU: compiles tests/native/geometry_check.cu with nvcc as host
code and runs it (see the file for what it checks)."""
import pathlib
import shutil
import subprocess

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]


def _nvcc():
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and pathlib.Path(c).exists():
            return c
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_gemv_work_split(tmp_path):
    exe = tmp_path / "geometry_check"
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
           "-I", str(ROOT / "include"), "-I", str(ROOT / "w4_weight_only_b200" / "csrc"),
           str(ROOT / "tests" / "native" / "geometry_check.cu"), "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and "geometry ok" in out.stdout, out.stdout[-2000:]
