"""Strength of the oracle pins: plausible mistakes planted in a copy of the
oracle's C source must each make tests/test_oracle_pins.py fail.

Every mutant is one textual change of oracle/nectar_oracle.c (or of the
oracle's Python side: parameter order, head selection) -- a dropped
term or factor, a wrong sign, a transposed operand, an off-by-one index --
applied to a scratch copy of the oracle package together with the pin tests
and their golden files; the copy builds its own library and the pins run
against it in a subprocess.  The committed oracle is never modified.  An
unmutated copy must pass, so a harness fault cannot pass for a detection."""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nectar_oracle.c")
PY = os.path.join(ROOT, "oracle", "__init__.py")

# (name, old text, new text): each old text occurs exactly once in the source
MUTANTS = [
    # exact attention, Eq. (3.1)
    ("alpha drops the max shift", "alpha[it] = (n > 0) ? M + log(l) : -INFINITY;",
     "alpha[it] = (n > 0) ? log(l) : -INFINITY;"),
    ("weights lose the scale", "double w = exp(scale * dot_bf16(q, Kh + j * d, d) - M);",
     "double w = exp(dot_bf16(q, Kh + j * d, d) - M);"),
    ("A is not normalised", "        for (int c = 0; c < d; ++c) out[c] /= l;\n", ""),
    ("dot product skips the last dim", "for (int c = 0; c < d; ++c) s += bf16_to_double(q[c])",
     "for (int c = 0; c < d - 1; ++c) s += bf16_to_double(q[c])"),
    # MLP, Eq. (3.6)
    ("SiLU sign", "return x / (1.0 + exp(-x));", "return x / (1.0 + exp(x));"),
    ("layer 0 drops its bias",
     "        const double *b0 = U0 + (int64_t)H * d;\n        for (int i = 0; i < H; ++i) {\n"
     "            double z = b0[i];",
     "        const double *b0 = U0 + (int64_t)H * d;\n        for (int i = 0; i < H; ++i) {\n"
     "            double z = 0.0;"),
    ("no re-injection of q",
     "                for (int c = 0; c < d; ++c) z += Vk[(int64_t)i * d + c] * q[c];\n"
     "                for (int j = 0; j < H; ++j) z += Uk",
     "                for (int j = 0; j < H; ++j) z += Uk"),
    ("U_k transposed", "z += Uk[(int64_t)i * H + j] * h[j];", "z += Uk[(int64_t)j * H + i] * h[j];"),
    ("readout gets an activation",
     "            for (int j = 0; j < H; ++j) z += W[(int64_t)o * H + j] * h[j];\n            y[o] = z;",
     "            for (int j = 0; j < H; ++j) z += W[(int64_t)o * H + j] * h[j];\n            y[o] = silu(z);"),
    ("readout bias dropped from the layout", "return P + (int64_t)dout * H + dout;",
     "return P + (int64_t)dout * H;"),
    # chain of a shared backbone (App. A.3)
    ("chain: U_k transposed", "z += Uk[(int64_t)i * Hp + j] * h[j];", "z += Uk[(int64_t)j * Hk + i] * h[j];"),
    ("chain: no re-injection of q",
     "                for (int c = 0; c < d; ++c) z += Vk[(int64_t)i * d + c] * q[c];\n"
     "                for (int j = 0; j < Hp; ++j)",
     "                for (int j = 0; j < Hp; ++j)"),
    # merge with exact causal local attention, Eqs. (3.4)-(3.5)
    ("causal set excludes the token itself", "int64_t v = (int64_t)pos + 1;", "int64_t v = (int64_t)pos;"),
    ("local_len ignored", "    if (v > len) v = len;\n", ""),
    ("document weight dropped from the numerator", "o[c] = wdoc * Adoc[it * d + c];",
     "o[c] = Adoc[it * d + c];"),
    ("document weight dropped from the denominator", "double den = wdoc;", "double den = 1.0;"),
    ("row mapped to the wrong token",
     "i = r % nq;\n        int64_t b = q_seq[i];\n        int64_t nv = visible_count(q_pos[i], local_len[b]);\n"
     "        const uint16_t *q = Q + it * d;\n        const uint16_t *Kb",
     "i = (r + 1) % nq;\n        int64_t b = q_seq[i];\n        int64_t nv = visible_count(q_pos[i], local_len[b]);\n"
     "        const uint16_t *q = Q + it * d;\n        const uint16_t *Kb"),
    # fit metrics, Eq. (C.1)
    ("RTE ratio inverted", "r_sum += log(num / den);", "r_sum += log(den / num);"),
    ("target MSE misses 1/d", "t_sum += num / d;", "t_sum += num;"),
    ("score error not squared", "s_sum += ds * ds;", "s_sum += ds;"),
]

# the same for the oracle's Python side (parameter order, head selection)
PY_MUTANTS = [
    ("flatten_net: U_k before V_k", "parts += [Vs[k][h], U[k][h], b[k][h]]", "parts += [U[k][h], Vs[k][h], b[k][h]]"),
    ("flatten_chain: U_k before V_k", "else [V[h], U[h], b[h]]", "else [U[h], V[h], b[h]]"),
    ("module_forward: heads in reverse", "X = wl.Q[l, hs].reshape(len(hs), wl.rows, wl.d)",
     "X = wl.Q[l, hs[::-1]].reshape(len(hs), wl.rows, wl.d)"),
    ("quadrature: W and Z swapped", "return cache_attn(W, Z, Q, scale)", "return cache_attn(Z, W, Q, scale)"),
    ("RTE summed over the wrong column", "float(out[:, 2].sum())", "float(out[:, 1].sum())"),
]


def _tree(base: str, source: str, py_source: str) -> str:
    """A scratch repository holding the oracle (with `source` as its C file
    and `py_source` as its Python module), the input generators, the pin
    tests and their golden files."""
    os.makedirs(os.path.join(base, "oracle"))
    with open(os.path.join(base, "oracle", "__init__.py"), "w") as f:
        f.write(py_source)
    with open(os.path.join(base, "oracle", "nectar_oracle.c"), "w") as f:
        f.write(source)
    shutil.copytree(os.path.join(ROOT, "nectar_inputs"), os.path.join(base, "nectar_inputs"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(base, "tests"))
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(base, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(base, "tests", "golden"))
    return base


def _run_pins(base: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, OMP_NUM_THREADS="2", PYTHONDONTWRITEBYTECODE="1")
    env.pop("PYTHONPATH", None)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join("tests", "test_oracle_pins.py")],
                          cwd=base, env=env, capture_output=True, text=True, timeout=900)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    with open(SRC) as f:
        source = f.read()
    with open(PY) as f:
        py_source = f.read()
    for name, old, _ in PY_MUTANTS:
        assert py_source.count(old) == 1, f"mutant '{name}': its text occurs {py_source.count(old)} times"
    for name, old, new in MUTANTS:
        assert source.count(old) == 1, f"mutant '{name}': its text occurs {source.count(old)} times"
        chk = subprocess.run(["gcc", "-fsyntax-only", "-std=c11", "-fopenmp", "-x", "c", "-"],
                             input=source.replace(old, new), capture_output=True, text=True)
        assert chk.returncode == 0, f"mutant '{name}' does not compile:\n{chk.stderr}"
    control = _run_pins(_tree(str(tmp_path / "control"), source, py_source))
    assert control.returncode == 0, "the unmutated copy must pass:\n" + control.stdout[-3000:]
    jobs = {}
    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, (os.cpu_count() or 2) // 2))) as ex:
        for k, (name, old, new) in enumerate(MUTANTS):
            base = _tree(str(tmp_path / f"m{k}"), source.replace(old, new), py_source)
            jobs[name] = ex.submit(_run_pins, base)
        for k, (name, old, new) in enumerate(PY_MUTANTS):
            base = _tree(str(tmp_path / f"p{k}"), source, py_source.replace(old, new))
            jobs[name] = ex.submit(_run_pins, base)
    survivors = [name for name, fut in jobs.items() if fut.result().returncode == 0]
    assert not survivors, f"mutants no pin catches: {survivors}"
    # a detection is a failed pin, not a crash or a collection error
    odd = [name for name, fut in jobs.items()
           if " failed" not in (fut.result().stdout.strip().splitlines() or [""])[-1]]
    assert not odd, f"mutants that ended without a failed pin: {odd}"
