"""The stream-K planners of the exact-attention kernels, checked on the CPU:
tests/host_plans.cu is linked against the library's own objects (no GPU is
touched) and counts by brute force, from the CTA-to-tile partition the
kernels use, what plan_decode, plan_tc and dec_smem_for_rows claim."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stream_k_plans(tmp_path):
    from long_context_attention_split_b200 import build
    try:
        nvcc = build.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not found")
    build.build()
    objs = [os.path.join(build.BUILD, f) for f in ("attn_decode.o", "attn_tc.o")]
    exe = str(tmp_path / "host_plans")
    cmd = [nvcc, *build.ARCH, "-std=c++17", "-O1", "-I", build.CSRC, os.path.join(ROOT, "tests", "host_plans.cu"),
           *objs, "-lcuda", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok "), r.stdout
    assert int(r.stdout.split()[1]) > 8000
