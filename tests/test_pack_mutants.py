"""Strength of the packing test: layout mistakes planted in a scratch copy of
csrc/module_layout.h must each make test_abi.test_pack_layout (the
independent reader of the tiled, swizzled weight blob) fail.

For each mistake the packer's translation unit (nectar_api.cu) is rebuilt
next to the mutated header, linked with the library's other objects into a
scratch libnectar.so, and the packing test runs against that library in a
subprocess.  The library's own sources and build are not touched."""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, old text, new text) in module_layout.h
LAYOUT_MUTANTS = [
    ("swizzle dropped", "((((c % 64) >> 3) ^ (r & 7)) << 3)", "((((c % 64) >> 3)) << 3)"),
    ("swizzle on the wrong row bits", "((((c % 64) >> 3) ^ (r & 7)) << 3)", "((((c % 64) >> 3) ^ (r & 3)) << 3)"),
    ("chunk stride of a ragged row tile", "static_cast<int64_t>(c) * tile_rows(rows, m)) * 64",
     "static_cast<int64_t>(c) * 128) * 64"),
    ("bias not padded to 64", "off += chunked_elems(H, hidden_k(H, kk)) + round64(H);",
     "off += chunked_elems(H, hidden_k(H, kk)) + H;"),
    ("score readout row not padded", "return out_w_off(H, depth) + (dout == 1 ? round64(H) : chunked_elems(kDm, H));",
     "return out_w_off(H, depth) + (dout == 1 ? H : chunked_elems(kDm, H));"),
]

_RUNNER = r"""
import importlib.util, sys
sys.path.insert(0, sys.argv[1])
import long_context_attention_split_b200 as nx
nx.LIB_PATH = sys.argv[2]
nx._lib = None
spec = importlib.util.spec_from_file_location("test_abi_copy", sys.argv[3])
t = importlib.util.module_from_spec(spec)
spec.loader.exec_module(t)
for widths, depth, hkv in [([64, 32], 2, 2), ([48], 3, 1), ([16, 208], 1, 3), ([272], 2, 1)]:
    try:
        t.test_pack_layout(widths, depth, hkv)
    except AssertionError as e:
        print("FAILED", widths, depth, hkv)
        sys.exit(1)
print("passed")
"""


def test_planted_layout_mistakes_fail_the_packing_test(tmp_path):
    from long_context_attention_split_b200 import build
    try:
        nvcc = build.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not found")
    build.build()
    with open(os.path.join(build.CSRC, "module_layout.h")) as f:
        header = f.read()
    with open(os.path.join(build.CSRC, "nectar_api.cu")) as f:
        api = f.read()
    others = [os.path.join(build.BUILD, o) for o in sorted(os.listdir(build.BUILD))
              if o.endswith(".o") and o != "nectar_api.o"]
    runner = tmp_path / "runner.py"
    runner.write_text(_RUNNER)

    def run(k, old, new):
        assert header.count(old) == 1, old
        d = tmp_path / f"m{k}"
        d.mkdir()
        # nectar_api.cu beside the mutated header: its quoted include finds that one first
        (d / "module_layout.h").write_text(header.replace(old, new))
        (d / "nectar_api.cu").write_text(api)
        obj, lib = str(d / "nectar_api.o"), str(d / "libnectar.so")
        r = subprocess.run([nvcc, *build.ARCH, *build.NVCC_FLAGS, "-c", str(d / "nectar_api.cu"), "-o", obj],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stdout + r.stderr
        r = subprocess.run([nvcc, *build.ARCH, "-shared", "-Xcompiler", "-fPIC", obj, *others, "-o", lib],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stdout + r.stderr
        return subprocess.run([sys.executable, str(runner), ROOT, lib, os.path.join(ROOT, "tests", "test_abi.py")],
                              capture_output=True, text=True, timeout=300)

    # the harness itself: the unmutated header must pass
    control = run("control", LAYOUT_MUTANTS[0][1], LAYOUT_MUTANTS[0][1])
    assert control.returncode == 0 and "passed" in control.stdout, control.stdout + control.stderr
    with cf.ThreadPoolExecutor(max_workers=5) as ex:
        futs = {name: ex.submit(run, k, old, new) for k, (name, old, new) in enumerate(LAYOUT_MUTANTS)}
    caught = lambda r: r.returncode != 0 and "FAILED" in r.stdout
    missed = [name for name, f in futs.items() if not caught(f.result())]
    # a run that ended without reaching the packing test (a crash while five
    # builds and loads ran side by side under a busy suite) runs again, alone
    names = [m[0] for m in LAYOUT_MUTANTS]
    missed = [name for name in missed if not caught(run(f"{names.index(name)}r", *LAYOUT_MUTANTS[names.index(name)][1:]))]
    assert not missed, f"layout mistakes the packing test misses: {missed}"
