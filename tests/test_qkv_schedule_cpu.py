"""The fused QKV kernel's tile schedule, checked on the host.

`tests/qkv_schedule_check.cu` includes the kernel source and checks, for a set
of shapes, that the runs the CTA pairs take in turn cover every tile exactly
once, keep each run inside one chunk and column, respect the balance bound,
and size the partial workspace as the combine reads it. Compiled with nvcc and
run on the CPU (no GPU call is made)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "linear_attention_diffusion_b200", "csrc")


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_qkv_schedule_covers_every_tile_once(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    exe = str(tmp_path / "qkv_schedule_check")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    os.path.join(HERE, "qkv_schedule_check.cu"), "-o", exe],
                   check=True, capture_output=True, timeout=600)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("ALL OK"), out.stdout
    # the three bench workloads' run lengths (chosen for balance)
    assert "B=4 N=1024 H=70 C=2240: L=2 " in out.stdout
    assert "B=1 N=16384 H=70 C=2240: L=8 " in out.stdout
    assert "B=1 N=32760 H=70 C=2240: L=16 " in out.stdout
