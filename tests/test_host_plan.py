"""Host-side launch planning (route plan, tile width, fused select, tensor-core switch, shared
memory sizes) checked over a grid of shapes, and the activation-shift rule over every finite bf16
magnitude, by a small host program built with nvcc."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not os.path.exists(NVCC) and shutil.which("nvcc") is None, reason="needs nvcc")
def test_launch_plans_cover_every_shape(tmp_path):
    exe = str(tmp_path / "plan_check")
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
                           "--expt-relaxed-constexpr",
                           "-I", os.path.join(ROOT, "decode_moe_layer_b200", "csrc"),
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "host", "plan_check.cu"), "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok")
