"""The algorithmic flops and bytes that gptq_kernel_times reports for each GEMM launch are a
closed form per output row (csrc/ktimes.cuh); a host-only checker compares them with a
brute-force count over every (i, j, k) of random small shapes and structure flags."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_gemm_work_counts_match_brute_force(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "kt_count_check")
    subprocess.run([nvcc, "-std=c++17", "-O1", "-Wno-deprecated-gpu-targets",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "post_weight_quantization_06_b200", "csrc"),
                    "-o", exe, os.path.join(ROOT, "tests", "kt_count_check.cu")],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    print(out.stdout)
    assert out.returncode == 0, out.stdout
    assert out.stdout.strip().endswith("0 of 3000 cases differ")
