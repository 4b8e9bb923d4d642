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


# (source file, name, old text, new text): planner mistakes the checker must catch
PLAN_MUTANTS = [
    ("attn_decode.cu", "S_max one short", "if (la - f + 1 > pl.S_max) pl.S_max = la - f + 1;",
     "if (la - f > pl.S_max) pl.S_max = la - f;"),
    ("attn_decode.cu", "C not clamped to the tile count", "  if (C > pl.total) C = pl.total;\n", ""),
    ("attn_tc.cu", "no whole round left for the stream-K part", "  if (best_s == 0 && rest != 0 && R > 0) R -= 1;\n",
     ""),
    ("attn_tc.cu", "lockstep balance ignored", "if (best_s > 0 && best * 10 > even * 11) best_s = 0;", ""),
    ("attn_tc.cu", "one partial slot per CTA",
     "pl.ws_bytes = static_cast<size_t>(pl.C) * 2 * kTcUnitRows", "pl.ws_bytes = static_cast<size_t>(pl.C) * 1 * kTcUnitRows"),
]


def test_planted_planner_mistakes_fail_the_checker(tmp_path):
    """Each mistake above, planted in a scratch copy of its source (the
    library's own files are not touched), makes tests/host_plans.cu fail."""
    import concurrent.futures as cf
    from long_context_attention_split_b200 import build
    try:
        nvcc = build.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not found")
    build.build()

    def run(k, fname, old, new):
        with open(os.path.join(build.CSRC, fname)) as f:
            src = f.read()
        assert src.count(old) == 1, (fname, old)
        d = tmp_path / f"m{k}"
        d.mkdir()
        mutated = d / fname
        mutated.write_text(src.replace(old, new))
        other = "attn_tc.o" if fname == "attn_decode.cu" else "attn_decode.o"
        exe = str(d / "host_plans")
        r = subprocess.run([nvcc, *build.ARCH, "-std=c++17", "-O1", "--expt-relaxed-constexpr", "-I", build.CSRC,
                            "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "host_plans.cu"),
                            str(mutated), os.path.join(build.BUILD, other), "-lcuda", "-o", exe],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stdout + r.stderr
        return subprocess.run([exe], capture_output=True, text=True, timeout=300)

    with cf.ThreadPoolExecutor(max_workers=4) as ex:
        futs = {name: ex.submit(run, k, fname, old, new) for k, (fname, name, old, new) in enumerate(PLAN_MUTANTS)}
    missed = [name for name, f in futs.items() if f.result().returncode == 0 or "FAIL" not in f.result().stdout]
    assert not missed, f"planner mistakes the checker misses: {missed}"
