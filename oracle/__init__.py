"""CPU oracle for the Nectar hot path -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline leg may
import this package.  The product path (``long_context_attention_split_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``nectar_oracle.c`` (plain C, IEEE double, OpenMP
over independent items only); this module builds it with gcc and marshals
numpy / torch CPU arrays into it.  Formulas follow "Nectar: Neural
Estimation of Cached-Token Attention via Regression" (Monteiro et al.):
Eq. (3.1) for the exact (alpha, A), Eq. (3.6) for the MLP, Eqs. (3.4)-(3.5)
for the merge with local tokens.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nectar_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile nectar_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        lib.oracle_cache_attn.argtypes = [I, I, I, ctypes.c_int, P, P, P, ctypes.c_double, P, P]
        lib.oracle_mlp_param_count.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.oracle_mlp_param_count.restype = I
        lib.oracle_mlp.argtypes = [I, I, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
        lib.oracle_chain_param_count.argtypes = [ctypes.c_int, ctypes.c_int, P, ctypes.c_int]
        lib.oracle_chain_param_count.restype = I
        lib.oracle_chain.argtypes = [I, I, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, P, P]
        lib.oracle_merge_local.argtypes = [I, I, I, ctypes.c_int, P, P, P, P, P, P, P, I, I, P,
                                           ctypes.c_double, P]
        lib.oracle_full_attention.argtypes = [I, I, I, I, ctypes.c_int, P, P, P, P, P, P, P, I, I, P,
                                              ctypes.c_double, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_fit_metrics.argtypes = [I, I, ctypes.c_int, P, P, P, P, P, P]
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_threads(t: int) -> None:
    _load().oracle_set_threads(int(t))


# --------------------------------------------------------------------------
# marshalling helpers
# --------------------------------------------------------------------------
def _bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor (any device) -> contiguous uint16 bit patterns."""
    import torch
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    assert x.dtype == torch.bfloat16, x.dtype
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f64(x) -> np.ndarray:
    import torch
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _i32(x) -> np.ndarray:
    import torch
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# public oracle functions
# --------------------------------------------------------------------------
def cache_attn(K, V, Q, scale: float):
    """Exact (alpha, A) of Eq. (3.1).

    K, V: bf16 [..., n, d]; Q: bf16 [..., rows, d] with the same leading
    (head) axes.  Returns (alpha [..., rows], A [..., rows, d]) in float64."""
    Kb, Vb, Qb = _bf16_bits(K), _bf16_bits(V), _bf16_bits(Q)
    n, d = Kb.shape[-2], Kb.shape[-1]
    rows = Qb.shape[-2]
    lead = Qb.shape[:-2]
    heads = int(np.prod(lead)) if lead else 1
    assert Kb.shape[:-2] == lead and Vb.shape == Kb.shape
    alpha = np.zeros(lead + (rows,), np.float64)
    A = np.zeros(lead + (rows, d), np.float64)
    _load().oracle_cache_attn(heads, n, rows, d, _p(Kb), _p(Vb), _p(Qb), float(scale),
                              _p(alpha), _p(A))
    return alpha, A


def mlp_param_count(d: int, depth: int, H: int, dout: int) -> int:
    return int(_load().oracle_mlp_param_count(d, depth, H, dout))


def flatten_net(net: dict, heads: Optional[List[int]] = None) -> np.ndarray:
    """One net's parameters (a dict from nectar_inputs.make_modules) in the
    oracle's plain row-major order, one row per KV head: [Hkv][P] float64."""
    import torch
    U, Vs, b, Wout, c = net["U"], net["V"], net["b"], net["Wout"], net["c"]
    hs = range(U[0].shape[0]) if heads is None else heads
    rows = []
    for h in hs:
        parts = [U[0][h], b[0][h]]
        for k in range(1, len(U)):
            parts += [Vs[k][h], U[k][h], b[k][h]]
        parts += [Wout[h], c[h]]
        rows.append(np.concatenate([p.detach().cpu().double().numpy().ravel() for p in parts]))
    return np.ascontiguousarray(np.stack(rows))


def mlp(params: np.ndarray, X, depth: int, H: int, dout: int):
    """Eq. (3.6) MLP.  params [units][P] (flatten_net order); X bf16 [units, rows, d].
    Returns Y [units, rows, dout] float64."""
    Xb = _bf16_bits(X)
    units, rows, d = Xb.shape
    P = mlp_param_count(d, depth, H, dout)
    params = _f64(params)
    assert params.shape == (units, P), (params.shape, units, P)
    Y = np.zeros((units, rows, dout), np.float64)
    _load().oracle_mlp(units, rows, d, depth, H, dout, _p(params), _p(Xb), _p(Y))
    return Y


def module_forward(wl, heads=None):
    """(a, A_theta) for every (l, h) of a workload (or a subset of layers
    given as `heads` = list of (l, h)).  Returns dicts keyed by (l, h):
    a [rows], A_theta [rows, d]."""
    out_a, out_A = {}, {}
    sel = heads if heads is not None else [(l, h) for l in range(wl.L) for h in range(wl.Hkv)]
    by_layer: Dict[int, List[int]] = {}
    for (l, h) in sel:
        by_layer.setdefault(l, []).append(h)
    for l, hs in by_layer.items():
        H = wl.widths[l]
        X = wl.Q[l, hs].reshape(len(hs), wl.rows, wl.d)
        for net, dout in (("score", 1), ("target", wl.d)):
            Y = mlp(flatten_net(wl.modules[l][net], hs), X, wl.depth, H, dout)
            for j, h in enumerate(hs):
                if net == "score":
                    out_a[(l, h)] = Y[j, :, 0]
                else:
                    out_A[(l, h)] = Y[j]
    return out_a, out_A


def flatten_chain(backbone: Optional[dict], net: dict, heads: Optional[List[int]] = None):
    """The parameters of one net with a shared backbone in front (dicts from
    nectar_inputs.make_modules_general), as the chain the oracle runs: the
    backbone's layers, then the branch's, then the readout.  Returns
    (params [Hkv][P] float64, per-layer widths)."""
    layers = []
    if backbone is not None:
        layers += [(backbone["U"][k], backbone["V"][k], backbone["b"][k]) for k in range(len(backbone["U"]))]
    layers += [(net["U"][k], net["V"][k], net["b"][k]) for k in range(len(net["U"]))]
    widths = [int(U.shape[1]) for (U, _, _) in layers]
    hs = range(net["Wout"].shape[0]) if heads is None else heads
    rows = []
    for h in hs:
        parts = []
        for k, (U, V, b) in enumerate(layers):
            # the chain's first layer sees only q (through U); later ones see
            # q through V and the previous layer through U
            assert (V is None) == (k == 0)
            parts += ([U[h], b[h]] if k == 0 else [V[h], U[h], b[h]])
        parts += [net["Wout"][h], net["c"][h]]
        rows.append(np.concatenate([p.detach().cpu().double().numpy().ravel() for p in parts]))
    return np.ascontiguousarray(np.stack(rows)), widths


def chain(params: np.ndarray, X, widths: List[int], dout: int):
    """A chain of Eq. (3.6) layers with per-layer widths, then the linear
    readout.  params [units][P] (flatten_chain order); X bf16 [units, rows, d].
    Returns Y [units, rows, dout] float64."""
    Xb = _bf16_bits(X)
    units, rows, d = Xb.shape
    W = np.ascontiguousarray(np.asarray(widths, dtype=np.int32))
    P = int(_load().oracle_chain_param_count(d, len(widths), _p(W), dout))
    params = _f64(params)
    assert params.shape == (units, P), (params.shape, units, P)
    Y = np.zeros((units, rows, dout), np.float64)
    _load().oracle_chain(units, rows, d, len(widths), _p(W), dout, _p(params), _p(Xb), _p(Y))
    return Y


def module_forward_general(mods, Q, heads=None):
    """(a, A_theta) of module sets with a shared backbone (depths
    (D_b, D_s, D_t), App. A.3; mods from nectar_inputs.make_modules_general):
    the score output is the chain backbone -> score branch -> readout, the
    target output the chain backbone -> target branch -> readout.
    Q bf16 [L][Hkv][G][nq][d].  Returns dicts keyed by (l, h): a [rows],
    A_theta [rows, d]."""
    L, Hkv, G, nq, d = Q.shape
    sel = heads if heads is not None else [(l, h) for l in range(L) for h in range(Hkv)]
    by_layer: Dict[int, List[int]] = {}
    for (l, h) in sel:
        by_layer.setdefault(l, []).append(h)
    out_a, out_A = {}, {}
    for l, hs in by_layer.items():
        X = Q[l, hs].reshape(len(hs), G * nq, d)
        bb = mods[l]["backbone"] if mods[l]["backbone"]["U"] else None
        for net, dout in (("score", 1), ("target", d)):
            params, widths = flatten_chain(bb, mods[l][net], hs)
            Y = chain(params, X, widths, dout)
            for j, h in enumerate(hs):
                if net == "score":
                    out_a[(l, h)] = Y[j, :, 0]
                else:
                    out_A[(l, h)] = Y[j]
    return out_a, out_A


def merge_local(a, Adoc, Q, q_seq, q_pos, Kloc, Vloc, local_len, scale: float):
    """Eqs. (3.4)-(3.5) merge.  a [heads, rows], Adoc [heads, rows, d] (float),
    Q bf16 [heads, rows, d]; Kloc, Vloc bf16 [heads, B, T, d].  Returns out
    [heads, rows, d] float64."""
    a, Adoc = _f64(a), _f64(Adoc)
    Qb, Kb, Vb = _bf16_bits(Q), _bf16_bits(Kloc), _bf16_bits(Vloc)
    heads, rows, d = Qb.shape
    B, T = Kb.shape[1], Kb.shape[2]
    qs, qp, ll = _i32(q_seq), _i32(q_pos), _i32(local_len)
    nq = qs.shape[0]
    assert rows % nq == 0 and a.shape == (heads, rows) and Adoc.shape == (heads, rows, d)
    out = np.zeros((heads, rows, d), np.float64)
    _load().oracle_merge_local(heads, rows, nq, d, _p(a), _p(Adoc), _p(Qb), _p(qs), _p(qp),
                               _p(Kb), _p(Vb), B, T, _p(ll), float(scale), _p(out))
    return out


def full_attention(K, V, Q, q_seq, q_pos, Kloc, Vloc, local_len, scale: float):
    """Left side of Eq. (3.4): one softmax over [document ; visible local]."""
    Kb, Vb, Qb = _bf16_bits(K), _bf16_bits(V), _bf16_bits(Q)
    Klb, Vlb = _bf16_bits(Kloc), _bf16_bits(Vloc)
    heads, n, d = Kb.shape
    rows = Qb.shape[1]
    B, T = Klb.shape[1], Klb.shape[2]
    qs, qp, ll = _i32(q_seq), _i32(q_pos), _i32(local_len)
    nq = qs.shape[0]
    out = np.zeros((heads, rows, d), np.float64)
    _load().oracle_full_attention(heads, n, rows, nq, d, _p(Kb), _p(Vb), _p(Qb), _p(qs), _p(qp),
                                  _p(Klb), _p(Vlb), B, T, _p(ll), float(scale), _p(out))
    return out


def quadrature_forward(W, Z, Q, scale: float):
    """Quadrature module of §2.4: a_theta(q) = log sum_j exp((W q)_j / sqrt d),
    A_theta(q) = softmax(W q / sqrt d)^T Z, with W, Z [..., p, d] the learned
    rows (initialised to the first p rows of K and V).  By its definition this
    is the exact attention of Eq. (3.1) over (W, Z), computed as such."""
    return cache_attn(W, Z, Q, scale)


def fit_metrics(alpha, A, a, At, Q):
    """Per (l, h) score MSE, target MSE (per element) and mean log error ratio
    of Eq. (C.1) (App. C.4); returns [heads, 3] float64 and the RTE (the sum
    of the last column).  alpha, a: [..., rows]; A, At: [..., rows, d];
    Q: bf16 [..., rows, d]."""
    al, aa = _f64(alpha), _f64(a)
    Ad, At_ = _f64(A), _f64(At)
    Qb = _bf16_bits(Q)
    rows, d = Ad.shape[-2], Ad.shape[-1]
    heads = int(np.prod(Ad.shape[:-2])) if Ad.ndim > 2 else 1
    out = np.zeros((heads, 3), np.float64)
    _load().oracle_fit_metrics(heads, rows, d, _p(al), _p(Ad), _p(aa), _p(At_), _p(Qb), _p(out))
    return out, float(out[:, 2].sum())
