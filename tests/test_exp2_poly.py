"""The software exp2 of the tensor-core softmax (exp2_poly in common.cuh):
its coefficients, read from the header, and its fp32 steps emulated in
numpy, against exact 2^x.  The bound is the polynomial's minimax error on
[-0.5, 0.5] (7.5e-5) plus fp32 rounding of the few operations, far below
the 2^-9 relative rounding of the bf16 softmax weights that follow."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "long_context_attention_split_b200", "csrc", "common.cuh")


def _coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1))) for i in range(4)]


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def exp2_poly_emulated(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(_f32(x), np.float32(-126.0))
    shifter = np.float32(12582912.0)
    j = _f32(x.astype(np.float64) + shifter)
    f = _f32(x.astype(np.float64) - _f32(j.astype(np.float64) - shifter))
    fma = lambda a, b, c: _f32(a.astype(np.float64) * b + c)     # fp32 FMA (exactly rounded once)
    pf = fma(fma(fma(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = pf.view(np.int32).astype(np.int64) + (j.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_match_the_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit", os.path.join(os.path.dirname(HDR), "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.remez(3)
    assert [float(v) for v in c] == [float(v) for v in _coeffs()]
    assert err < 8e-5


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.5, 127, 2_000_001), np.arange(-125, 128, dtype=np.float64),
                        np.arange(-125, 127) + 0.5, [0.0, -0.0, 1e-8, -1e-8]])
    got = exp2_poly_emulated(x).astype(np.float64)
    ref = np.exp2(_f32(x).astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.0e-4, rel.max()
    # the last half unit above the clamp lands in the subnormal range, where
    # the exponent trick drops the implicit bit: still within 2e-4 (and the
    # value, ~1e-38, is nothing next to a softmax row maximum of 1)
    edge = np.linspace(-126, -125.5, 10001)
    rel = np.abs(exp2_poly_emulated(edge).astype(np.float64) / np.exp2(edge) - 1)
    assert rel.max() < 2.0e-4, rel.max()


def test_integers_and_clamp():
    n = np.arange(-125, 128, dtype=np.float64)
    got = exp2_poly_emulated(n).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(n) - 1) < 1e-4)
    # below the clamp the result stays a tiny positive number
    tiny = exp2_poly_emulated(np.array([-200.0, -1e30, -np.inf]))
    assert np.all((tiny > 0) & (tiny < 1.2e-38 * 1.01))
