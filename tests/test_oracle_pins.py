"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks one oracle function against brute force on tiny inputs,
a closed form, an invariant of the mathematics, an independent library
routine (torch fp64 on the CPU), or a value printed on the Nectar pages
("Nectar: Neural Estimation of Cached-Token Attention via Regression").
The cases are chosen so that a dropped term, a wrong sign, a wrong index or
a transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from nectar_inputs import (capacity, kv_cache_bytes, make_workload, module_params_per_head,
                           nonuniform_widths)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def f64(x):
    return x.to(torch.float64)


def rand_bf16(gen, *shape, std=1.0):
    return (torch.randn(*shape, generator=gen) * std).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# (i) exact cached-token attention, Eq. (3.1)
# ---------------------------------------------------------------------------
def brute_alpha_A(q, K, V, scale):
    """Direct sums without any max shift, with math.fsum (tiny inputs)."""
    qd = [float(x) for x in q]
    s = [scale * math.fsum(qd[c] * float(K[j, c]) for c in range(K.shape[1]))
         for j in range(K.shape[0])]
    e = [math.exp(x) for x in s]
    Z = math.fsum(e)
    A = [math.fsum(e[j] * float(V[j, c]) for j in range(K.shape[0])) / Z
         for c in range(V.shape[1])]
    return math.log(Z), np.array(A)


@pytest.mark.parametrize("n,d,rows", [(1, 4, 2), (5, 3, 3), (16, 8, 4), (11, 7, 1)])
def test_cache_attn_brute_force(n, d, rows):
    g = torch.Generator().manual_seed(100 + n * d)
    K, V, Q = rand_bf16(g, 2, n, d), rand_bf16(g, 2, n, d), rand_bf16(g, 2, rows, d)
    scale = 1.0 / math.sqrt(d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    for h in range(2):
        for r in range(rows):
            ba, bA = brute_alpha_A(f64(Q[h, r]), f64(K[h]), f64(V[h]), scale)
            assert abs(alpha[h, r] - ba) < 1e-12
            np.testing.assert_allclose(A[h, r], bA, rtol=0, atol=1e-12)


def test_cache_attn_closed_forms():
    g = torch.Generator().manual_seed(7)
    d, scale = 128, 1.0 / math.sqrt(128)
    # n = 1: alpha = s_1, A = v_1
    K, V, Q = rand_bf16(g, 1, 1, d), rand_bf16(g, 1, 1, d), rand_bf16(g, 1, 3, d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    s = (f64(Q[0]) @ f64(K[0, 0])) * scale
    np.testing.assert_allclose(alpha[0], s.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(A[0], np.broadcast_to(f64(V[0, 0]).numpy(), (3, d)))
    # all keys equal: alpha = s + log n, A = mean(v)
    n = 37
    K = rand_bf16(g, 1, 1, d).expand(1, n, d).contiguous()
    V = rand_bf16(g, 1, n, d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    s = (f64(Q[0]) @ f64(K[0, 0])) * scale
    np.testing.assert_allclose(alpha[0], (s + math.log(n)).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(A[0], np.broadcast_to(f64(V[0]).mean(0).numpy(), (3, d)),
                               rtol=0, atol=1e-13)
    # q = 0: alpha = log n exactly, A = mean(v)
    Q0 = torch.zeros(1, 2, d, dtype=torch.bfloat16)
    K = rand_bf16(g, 1, n, d)
    alpha, A = oracle.cache_attn(K, V, Q0, scale)
    assert np.all(alpha == math.log(n))
    np.testing.assert_allclose(A[0], np.broadcast_to(f64(V[0]).mean(0).numpy(), (2, d)),
                               rtol=0, atol=1e-13)


def test_cache_attn_matches_torch_fp64():
    g = torch.Generator().manual_seed(11)
    heads, n, rows, d = 3, 300, 5, 128
    K, V, Q = rand_bf16(g, heads, n, d), rand_bf16(g, heads, n, d, std=2.0), rand_bf16(g, heads, rows, d)
    scale = 1.0 / math.sqrt(d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    S = torch.einsum("hrd,hnd->hrn", f64(Q), f64(K)) * scale
    ref_alpha = torch.logsumexp(S, dim=-1)
    ref_A = torch.softmax(S, dim=-1) @ f64(V)
    np.testing.assert_allclose(alpha, ref_alpha.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(A, ref_A.numpy(), rtol=0, atol=1e-12)


def test_cache_attn_invariants():
    """max_j s_j <= alpha <= max_j s_j + log n; A inside the per-coordinate
    range of the v_j (a consequence of lying in their convex hull)."""
    g = torch.Generator().manual_seed(12)
    heads, n, rows, d = 2, 513, 6, 128
    K, V, Q = rand_bf16(g, heads, n, d, std=1.7), rand_bf16(g, heads, n, d), rand_bf16(g, heads, rows, d)
    scale = 1.0 / math.sqrt(d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    S = (torch.einsum("hrd,hnd->hrn", f64(Q), f64(K)) * scale).numpy()
    smax = S.max(-1)
    assert np.all(alpha >= smax - 1e-12) and np.all(alpha <= smax + math.log(n) + 1e-12)
    vmin, vmax = f64(V).amin(1).numpy(), f64(V).amax(1).numpy()
    assert np.all(A >= vmin[:, None, :] - 1e-12) and np.all(A <= vmax[:, None, :] + 1e-12)


@pytest.mark.parametrize("parts", [2, 3, 8])
def test_cache_attn_split_lse_merge(parts):
    """Splitting the cache and LSE-merging the parts equals the unsplit
    result: the grouping of the softmax sum behind Eq. (3.4)."""
    g = torch.Generator().manual_seed(20 + parts)
    n, rows, d = 777, 4, 128
    K, V, Q = rand_bf16(g, 1, n, d), rand_bf16(g, 1, n, d), rand_bf16(g, 1, rows, d)
    scale = 1.0 / math.sqrt(d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    cuts = sorted(torch.randperm(n - 1, generator=g)[: parts - 1].add(1).tolist())
    bounds = [0] + cuts + [n]
    pa, pA = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        a_p, A_p = oracle.cache_attn(K[:, lo:hi].contiguous(), V[:, lo:hi].contiguous(), Q, scale)
        pa.append(a_p[0]); pA.append(A_p[0])
    pa, pA = np.stack(pa), np.stack(pA)          # [parts, rows], [parts, rows, d]
    M = pa.max(0)
    w = np.exp(pa - M)
    merged_alpha = M + np.log(w.sum(0))
    merged_A = (w[..., None] * pA).sum(0) / w.sum(0)[..., None]
    np.testing.assert_allclose(merged_alpha, alpha[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(merged_A, A[0], rtol=0, atol=1e-12)


def test_cache_attn_low_temperature_limit():
    """beta^{-1} log sum_j e^{beta s_j} -> max_j s_j  (App. B), with
    0 <= alpha(beta q)/beta - max_j s_j <= log(n)/beta."""
    g = torch.Generator().manual_seed(31)
    n, d = 200, 128
    K, V = rand_bf16(g, 1, n, d), rand_bf16(g, 1, n, d)
    q = rand_bf16(g, 1, 1, d)
    scale = 1.0 / math.sqrt(d)
    smax = float((f64(q[0]) @ f64(K[0]).T).max()) * scale
    prev = None
    for beta in [1, 4, 16, 64, 256]:          # powers of two: beta*q exact in bf16
        a, _ = oracle.cache_attn(K, V, (q.float() * beta).to(torch.bfloat16), scale)
        gap = a[0, 0] / beta - smax
        assert -1e-12 <= gap <= math.log(n) / beta + 1e-12
        if prev is not None:
            assert gap <= prev + 1e-12
        prev = gap
    assert prev < 0.05


# ---------------------------------------------------------------------------
# (ii) MLP with input re-injection, Eq. (3.6)
# ---------------------------------------------------------------------------
def rand_net(g, hkv, H, d, dout, depth=2, zero=False):
    def w(*shape, std):
        t = torch.randn(*shape, generator=g) * std
        return (t * 0 if zero else t).to(torch.bfloat16)
    U = [w(hkv, H, d, std=0.3)] + [w(hkv, H, H, std=0.3) for _ in range(1, depth)]
    Vs = [None] + [w(hkv, H, d, std=0.3) for _ in range(1, depth)]
    b = [w(hkv, H, std=0.5) for _ in range(depth)]
    Wout = w(hkv, dout, H, std=0.3)
    c = (torch.randn(hkv, dout, generator=g)).to(torch.bfloat16)
    return dict(U=U, V=Vs, b=b, Wout=Wout, c=c, H=H, dout=dout)


def torch_mlp(net, X, h):
    """Independent fp64 forward with torch.nn.functional.linear + silu."""
    q = f64(X)
    z = F.linear(q, f64(net["U"][0][h]), f64(net["b"][0][h]))
    hid = F.silu(z)
    for k in range(1, len(net["U"])):
        z = F.linear(q, f64(net["V"][k][h])) + F.linear(hid, f64(net["U"][k][h]), f64(net["b"][k][h]))
        hid = F.silu(z)
    return F.linear(hid, f64(net["Wout"][h]), f64(net["c"][h]))


@pytest.mark.parametrize("depth,H,dout", [(2, 64, 1), (2, 48, 128), (3, 32, 128), (1, 16, 1)])
def test_mlp_matches_torch_fp64(depth, H, dout):
    g = torch.Generator().manual_seed(40 + depth * H + dout)
    hkv, rows, d = 3, 5, 128
    net = rand_net(g, hkv, H, d, dout, depth)
    X = rand_bf16(g, hkv, rows, d)
    Y = oracle.mlp(oracle.flatten_net(net), X, depth, H, dout)
    for h in range(hkv):
        np.testing.assert_allclose(Y[h], torch_mlp(net, X[h], h).numpy(), rtol=1e-12, atol=1e-12)


def test_mlp_brute_force_tiny():
    """H = 4, d = 4, depth 2, pure Python loops with math.exp."""
    g = torch.Generator().manual_seed(50)
    H, d, dout = 4, 4, 3
    net = rand_net(g, 1, H, d, dout, 2)
    X = rand_bf16(g, 1, 2, d)
    Y = oracle.mlp(oracle.flatten_net(net), X, 2, H, dout)

    def silu(x):
        return x / (1.0 + math.exp(-x))

    def m(t):
        return f64(t).tolist()
    U0, b0, V1, U1, b1 = m(net["U"][0][0]), m(net["b"][0][0]), m(net["V"][1][0]), m(net["U"][1][0]), m(net["b"][1][0])
    W, c = m(net["Wout"][0]), m(net["c"][0])
    for r in range(2):
        q = m(X[0, r])
        h0 = [silu(b0[i] + sum(U0[i][k] * q[k] for k in range(d))) for i in range(H)]
        h1 = [silu(b1[i] + sum(V1[i][k] * q[k] for k in range(d)) + sum(U1[i][j] * h0[j] for j in range(H)))
              for i in range(H)]
        y = [c[o] + sum(W[o][j] * h1[j] for j in range(H)) for o in range(dout)]
        np.testing.assert_allclose(Y[0, r], y, rtol=1e-13, atol=1e-13)


def test_mlp_special_cases():
    g = torch.Generator().manual_seed(51)
    H, d, dout = 32, 128, 128
    X = rand_bf16(g, 2, 3, d)
    # all weights and biases zero except the readout bias: output = c
    net = rand_net(g, 2, H, d, dout, zero=True)
    net["c"] = rand_bf16(g, 2, dout)
    Y = oracle.mlp(oracle.flatten_net(net), X, 2, H, dout)
    np.testing.assert_array_equal(Y, np.broadcast_to(f64(net["c"]).numpy()[:, None, :], Y.shape))
    # U = V = 0: h_k = SiLU(b_k), output = W_out SiLU(b_1) + c, for any q
    net = rand_net(g, 2, H, d, dout)
    for k in range(2):
        net["U"][k] = torch.zeros_like(net["U"][k])
        if net["V"][k] is not None:
            net["V"][k] = torch.zeros_like(net["V"][k])
    Y = oracle.mlp(oracle.flatten_net(net), X, 2, H, dout)
    for h in range(2):
        b1 = f64(net["b"][1][h]).numpy()
        h1 = b1 / (1.0 + np.exp(-b1))
        ref = f64(net["Wout"][h]).numpy() @ h1 + f64(net["c"][h]).numpy()
        np.testing.assert_allclose(Y[h], np.broadcast_to(ref, (3, dout)), rtol=1e-13, atol=1e-13)


def test_module_forward_on_workload():
    """Workload-level wrapper routes each (l, h) to its own weights."""
    wl = make_workload("toy", L=2, Hkv=2, G=2, n=64, T=8, nq=8, H=32)
    a, A = oracle.module_forward(wl)
    for (l, h) in [(0, 0), (1, 1), (0, 1)]:
        X = wl.Q[l, h].reshape(wl.rows, wl.d)
        np.testing.assert_allclose(a[(l, h)], torch_mlp(wl.modules[l]["score"], X, h)[:, 0].numpy(),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(A[(l, h)], torch_mlp(wl.modules[l]["target"], X, h).numpy(),
                                   rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# (iii) merge with exact local attention, Eqs. (3.4)-(3.5)
# ---------------------------------------------------------------------------
def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_merge_worked_example():
    """§2.2: doc mass 9 / readout 2, local mass 3 / readout 10 -> 4."""
    (mass_doc, read_doc, mass_loc, read_loc, expected), = [list(map(float, r)) for r in
                                                          read_golden("worked_example.txt")]
    # one local token with q.k = 1 and scale = log(3) gives e^{s} = 3;
    # three tokens with s = 0 give the same mass.  d = 1.
    for T, scale, kval in [(1, math.log(mass_loc), 1.0), (3, 0.0, 1.0)]:
        Q = bf16([[[1.0]]])
        Kloc = bf16(np.full((1, 1, T, 1), kval))
        Vloc = bf16(np.full((1, 1, T, 1), read_loc))
        out = oracle.merge_local(np.array([[math.log(mass_doc)]]), np.array([[[read_doc]]]), Q,
                                 [0], [T - 1], Kloc, Vloc, [T], scale)
        assert abs(out[0, 0, 0] - expected) < 1e-14


def test_merge_gate_form():
    """g = sigmoid(a - log Z_local), out = g A + (1 - g) A_local, Z_local > 0."""
    g = torch.Generator().manual_seed(60)
    d, T = 128, 9
    Q, Kl, Vl = rand_bf16(g, 1, 1, d), rand_bf16(g, 1, 1, T, d), rand_bf16(g, 1, 1, T, d)
    a = np.array([[0.7]])
    A = np.random.default_rng(0).normal(size=(1, 1, d))
    scale = 1 / math.sqrt(d)
    out = oracle.merge_local(a, A, Q, [0], [T - 1], Kl, Vl, [T], scale)
    s = (f64(Kl[0, 0]) @ f64(Q[0, 0])).numpy() * scale
    Z = math.fsum(np.exp(s))
    A_loc = (np.exp(s)[:, None] * f64(Vl[0, 0]).numpy()).sum(0) / Z
    gate = 1.0 / (1.0 + math.exp(-(a[0, 0] - math.log(Z))))
    np.testing.assert_allclose(out[0, 0], gate * A[0, 0] + (1 - gate) * A_loc, rtol=0, atol=1e-13)


def sdpa_full(K, V, Q, q_seq, q_pos, Kloc, Vloc, local_len, scale):
    """torch SDPA in fp64 over [doc ; local] with an explicit boolean mask."""
    heads, n, d = K.shape
    rows = Q.shape[1]
    nq = len(q_seq)
    B, T = Kloc.shape[1], Kloc.shape[2]
    outs = []
    for hd in range(heads):
        for r in range(rows):
            i = r % nq
            b = q_seq[i]
            keys = torch.cat([f64(K[hd]), f64(Kloc[hd, b])])
            vals = torch.cat([f64(V[hd]), f64(Vloc[hd, b])])
            mask = torch.ones(n + T, dtype=torch.bool)
            loc = torch.arange(T)
            mask[n:] = (loc <= q_pos[i]) & (loc < local_len[b])
            o = F.scaled_dot_product_attention(f64(Q[hd, r])[None, None], keys[None], vals[None],
                                               attn_mask=mask[None, None], scale=scale)
            outs.append(o[0, 0])
    return torch.stack(outs).reshape(heads, rows, d).numpy()


def test_merge_of_exact_equals_full_attention():
    """Eq. (3.4) is exact: plugging the exact (alpha, A) into the merge gives
    full attention over document + visible local tokens (checked against
    the oracle's own one-softmax version and against torch SDPA)."""
    g = torch.Generator().manual_seed(70)
    heads, n, d, B, T, nq, G = 2, 150, 128, 3, 10, 4, 2
    K, V = rand_bf16(g, heads, n, d), rand_bf16(g, heads, n, d)
    Kl, Vl = rand_bf16(g, heads, B, T, d, std=1.5), rand_bf16(g, heads, B, T, d)
    Q = rand_bf16(g, heads, G * nq, d)
    q_seq, q_pos, local_len = [0, 1, 2, 1], [0, 9, 4, 3], [T, 7, 5]
    scale = 1 / math.sqrt(d)
    alpha, A = oracle.cache_attn(K, V, Q, scale)
    merged = oracle.merge_local(alpha, A, Q, q_seq, q_pos, Kl, Vl, local_len, scale)
    full = oracle.full_attention(K, V, Q, q_seq, q_pos, Kl, Vl, local_len, scale)
    ref = sdpa_full(K, V, Q, q_seq, q_pos, Kl, Vl, local_len, scale)
    np.testing.assert_allclose(full, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(merged, full, rtol=0, atol=1e-12)


def test_merge_mask_edges():
    g = torch.Generator().manual_seed(80)
    d, T, B = 128, 6, 4
    Q = rand_bf16(g, 1, 4, d)
    Kl, Vl = rand_bf16(g, 1, B, T, d), rand_bf16(g, 1, B, T, d)
    a = np.array([[0.3, -1.0, 2.0, 0.0]])
    A = np.random.default_rng(1).normal(size=(1, 4, d))
    scale = 1 / math.sqrt(d)
    # seq 0: q_pos 0 -> sees token 0 only; seq 1: local_len 1; seq 2: full
    # T_max; seq 3: local_len 0 -> out = A.
    q_seq, q_pos, local_len = [0, 1, 2, 3], [0, 5, T - 1, 2], [T, 1, T, 0]
    out = oracle.merge_local(a, A, Q, q_seq, q_pos, Kl, Vl, local_len, scale)
    for r, nvis in enumerate([1, 1, T, 0]):
        b = q_seq[r]
        s = (f64(Kl[0, b, :nvis]) @ f64(Q[0, r])).numpy() * scale
        w = np.concatenate([[a[0, r]], s])
        m = w.max()
        e = np.exp(w - m)
        vals = np.concatenate([A[0, r][None], f64(Vl[0, b, :nvis]).numpy()])
        np.testing.assert_allclose(out[0, r], (e[:, None] * vals).sum(0) / e.sum(), rtol=0, atol=1e-13)
    np.testing.assert_array_equal(out[0, 3], A[0, 3])


# ---------------------------------------------------------------------------
# sizing formulas against Table 9 and the capacity definition
# ---------------------------------------------------------------------------
def test_table9_storage():
    """Footprint 2nLHd x 2 B at n = 62000 and rho x footprint (App. A, Table 9)."""
    for name, L, Hkv, kv_gb, m2, m5, m10 in read_golden("table9_storage.txt"):
        kv = kv_cache_bytes(62000, int(L), int(Hkv), 128)
        assert round(kv / 1e9, 2) == float(kv_gb), name
        for rho, mb in [(0.02, m2), (0.05, m5), (0.10, m10)]:
            # the table prints whole MB and is not rounded consistently
            # (355.5 MB appears as 355): allow its 1 MB print precision
            assert abs(rho * kv / 1e6 - float(mb)) < 1.0, (name, rho)


def test_capacity_and_widths():
    # parameter count of a (score, target) pair at d = 128, depth 2
    for H in [16, 256, 512, 768]:
        assert module_params_per_head(H) == 2 * H * H + 645 * H + 129
        assert oracle.mlp_param_count(128, 2, H, 1) + oracle.mlp_param_count(128, 2, H, 128) \
            == module_params_per_head(H)
    assert abs(capacity(512, 32768) - 0.1019) < 1e-4
    # non-uniform widths: edge layers carry 1.5x the parameters, total = rho*2nd*L
    for rho in [0.01, 0.05, 0.10]:
        w = nonuniform_widths(rho, 32, 65536)
        assert all(x % 16 == 0 for x in w)
        total = sum(module_params_per_head(x) for x in w)
        assert abs(total / (rho * 2 * 65536 * 128 * 32) - 1) < 0.04
        assert w[0] > w[10] and w[0] == w[31] and w[4] == w[27]


# ---------------------------------------------------------------------------
# next rows: the Quadrature module (§2.4) and the fitting metrics (App. C.4)
# ---------------------------------------------------------------------------
def test_quadrature_is_attention_over_the_first_p_rows():
    """§2.4: a_theta = log sum_j exp((W q)_j / sqrt d), A_theta = softmax(.)^T Z,
    W, Z initialised to the first p rows of K, V -- brute force with fsum."""
    g = torch.Generator().manual_seed(77)
    n, p, d, rows = 12, 5, 6, 3
    K, V, Q = rand_bf16(g, 2, n, d), rand_bf16(g, 2, n, d), rand_bf16(g, 2, rows, d)
    W, Z = K[:, :p].contiguous(), V[:, :p].contiguous()
    a, At = oracle.quadrature_forward(W, Z, Q, 1 / math.sqrt(d))
    for h in range(2):
        for r in range(rows):
            ba, bA = brute_alpha_A(f64(Q[h, r]), f64(K[h, :p]), f64(V[h, :p]), 1 / math.sqrt(d))
            assert abs(a[h, r] - ba) < 1e-12
            assert np.abs(At[h, r] - bA).max() < 1e-12
    # p = 1: the softmax has one term, A_theta = z_1, a_theta = w_1 . q / sqrt d
    a1, At1 = oracle.quadrature_forward(K[:, :1].contiguous(), V[:, :1].contiguous(), Q, 1 / math.sqrt(d))
    assert np.abs(At1 - f64(V[:, :1]).numpy()).max() == 0.0
    s = (f64(Q) @ f64(K[:, :1]).transpose(1, 2)).squeeze(-1) / math.sqrt(d)
    assert np.abs(a1 - s.numpy()).max() < 1e-12


def test_fit_metrics_worked_example():
    """d = 2, one row: A = (0, 0), A_theta = (3, 4), q = (1, 0), alpha = 1,
    a = 3: score MSE 4, target MSE (9 + 16) / 2, RTE term log(25 / 1)."""
    A = np.zeros((1, 1, 2))
    At = np.array([[[3.0, 4.0]]])
    Q = bf16([[[1.0, 0.0]]])
    out, rte = oracle.fit_metrics(np.array([[1.0]]), A, np.array([[3.0]]), At, Q)
    assert out[0, 0] == 4.0 and out[0, 1] == 12.5
    assert abs(out[0, 2] - math.log(25.0)) < 1e-15 and abs(rte - math.log(25.0)) < 1e-15


def test_fit_metrics_special_cases_and_scaling():
    g = torch.Generator().manual_seed(5)
    heads, rows, d = 3, 7, 8
    alpha = torch.randn(heads, rows, generator=g, dtype=torch.float64)
    A = torch.randn(heads, rows, d, generator=g, dtype=torch.float64)
    Q = rand_bf16(g, heads, rows, d)
    E = torch.randn(heads, rows, d, generator=g, dtype=torch.float64)
    # a perfect module: both MSEs 0, every log ratio -inf
    out, _ = oracle.fit_metrics(alpha, A, alpha, A, Q)
    assert np.all(out[:, :2] == 0.0) and np.all(np.isneginf(out[:, 2]))
    # A_theta = q (the baseline of Eq. (C.1)): every log ratio is exactly 0
    out, rte = oracle.fit_metrics(alpha, A, alpha, f64(Q), Q)
    assert np.all(out[:, 2] == 0.0) and rte == 0.0
    # scaling the error by c scales the target MSE by c^2 and shifts each
    # log ratio by log c^2; the score MSE of a + c is c^2
    out1, rte1 = oracle.fit_metrics(alpha, A, alpha + 0.5, A + E, Q)
    out3, rte3 = oracle.fit_metrics(alpha, A, alpha + 1.5, A + 3.0 * E, Q)
    assert np.allclose(out1[:, 0], 0.25, rtol=0, atol=1e-15) and np.allclose(out3[:, 0], 2.25, rtol=0, atol=1e-15)
    assert np.allclose(out3[:, 1], 9.0 * out1[:, 1], rtol=1e-12)
    assert np.allclose(out3[:, 2], out1[:, 2] + math.log(9.0), rtol=0, atol=1e-12)
    assert abs(rte3 - (rte1 + heads * math.log(9.0))) < 1e-10
    # heads are independent: the metrics of a head do not see the others
    out_h, _ = oracle.fit_metrics(alpha[1:2], A[1:2], alpha[1:2] + 0.5, A[1:2] + E[1:2], Q[1:2])
    assert np.array_equal(out_h[0], out1[1])


# ---------------------------------------------------------------------------
# (ii) with a shared backbone: depths (D_b, D_s, D_t) and per-net widths
# (App. A.3, Eq. (3.6)).  The oracle runs each net as one chain (backbone
# layers, then the branch, then the readout).
# ---------------------------------------------------------------------------
def _general(L, Hkv, d, depths, wb, ws, wt, seed):
    from nectar_inputs import make_modules_general
    return make_modules_general(L, Hkv, d, seed, "cpu", depths, wb, ws, wt)


def _torch_general_forward(mods, Q):
    """The backbone run once with torch fp64 linear + silu, its last state
    handed to both branches (an independent implementation)."""
    L, Hkv, G, nq, d = Q.shape
    a, A = {}, {}
    for l in range(L):
        for h in range(Hkv):
            q = Q[l, h].reshape(G * nq, d).double()
            bb = mods[l]["backbone"]
            x = None
            for k in range(len(bb["U"])):
                z = F.linear(q, bb["U"][k][h].double(), bb["b"][k][h].double()) if k == 0 else \
                    F.linear(q, bb["V"][k][h].double()) + F.linear(x, bb["U"][k][h].double(), bb["b"][k][h].double())
                x = F.silu(z)
            outs = []
            for net in ("score", "target"):
                nt = mods[l][net]
                y = x
                for k in range(len(nt["U"])):
                    if nt["V"][k] is None:
                        z = F.linear(q, nt["U"][k][h].double(), nt["b"][k][h].double())
                    else:
                        z = F.linear(q, nt["V"][k][h].double()) + F.linear(y, nt["U"][k][h].double(),
                                                                          nt["b"][k][h].double())
                    y = F.silu(z)
                outs.append(F.linear(y, nt["Wout"][h].double(), nt["c"][h].double()).numpy())
            a[(l, h)] = outs[0][:, 0]
            A[(l, h)] = outs[1]
    return a, A


def test_general_module_without_backbone_is_the_separate_nets():
    # D_b = 0, equal widths: the chain oracle gives the (pinned) per-net MLP
    wl = make_workload("toy", L=2, Hkv=2, G=2, n=16, nq=3, with_local=False, with_modules=True,
                       widths=[32, 48], seed=5)
    mods = _general(2, 2, 128, (0, 2, 2), [0, 0], [32, 48], [32, 48], seed=5)
    a, A = oracle.module_forward_general(mods, wl.Q)
    a0, A0 = oracle.module_forward(wl)
    for key in a0:
        np.testing.assert_array_equal(a[key], a0[key])
        np.testing.assert_array_equal(A[key], A0[key])


@pytest.mark.parametrize("depths,wb,ws,wt", [((2, 1, 2), [48, 32], [32, 16], [16, 64]),
                                            ((0, 2, 3), [0, 0], [16, 48], [64, 32]),
                                            ((1, 1, 1), [64, 16], [32, 32], [48, 16])])
def test_general_module_against_torch(depths, wb, ws, wt):
    g = torch.Generator().manual_seed(7)
    Q = torch.randn(2, 2, 2, 3, 128, generator=g).to(torch.bfloat16)
    mods = _general(2, 2, 128, depths, wb, ws, wt, seed=11)
    a, A = oracle.module_forward_general(mods, Q)
    ta, tA = _torch_general_forward(mods, Q)
    for key in a:
        np.testing.assert_allclose(a[key], ta[key], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(A[key], tA[key], rtol=1e-12, atol=1e-12)


def test_general_module_brute_force_tiny():
    # d = 4, widths 3 / 2 / 5, depths (2, 1, 2): plain Python with math.fsum
    d = 4
    g = torch.Generator().manual_seed(3)
    Q = torch.randn(1, 1, 1, 2, d, generator=g).to(torch.bfloat16)
    mods = _general(1, 1, d, (2, 1, 2), [3], [2], [5], seed=13)
    a, A = oracle.module_forward_general(mods, Q)

    def silu(z):
        return z / (1.0 + math.exp(-z))

    def lin(W, x, b=None):
        W = W.double().tolist()
        out = [math.fsum(W[i][j] * x[j] for j in range(len(x))) for i in range(len(W))]
        if b is not None:
            out = [o + float(bb) for o, bb in zip(out, b.double().tolist())]
        return out

    for t in range(2):
        q = Q[0, 0, 0, t].double().tolist()
        bb = mods[0]["backbone"]
        x = [silu(z) for z in lin(bb["U"][0][0], q, bb["b"][0][0])]
        x = [silu(u + v) for u, v in zip(lin(bb["V"][1][0], q), lin(bb["U"][1][0], x, bb["b"][1][0]))]
        res = []
        for net in ("score", "target"):
            nt = mods[0][net]
            y = x
            for k in range(len(nt["U"])):
                y = [silu(u + v) for u, v in zip(lin(nt["V"][k][0], q), lin(nt["U"][k][0], y, nt["b"][k][0]))]
            res.append(lin(nt["Wout"][0], y, nt["c"][0]))
        assert abs(a[(0, 0)][t] - res[0][0]) <= 1e-12
        np.testing.assert_allclose(A[(0, 0)][t], res[1], rtol=0, atol=1e-12)


def test_general_module_zero_weights_closed_form():
    # U = V = 0: every layer is SiLU of its bias; the readout is W_out SiLU(b_last) + c
    mods = _general(1, 2, 128, (2, 1, 2), [32], [16], [48], seed=17)
    for part in ("backbone", "score", "target"):
        for k in range(len(mods[0][part]["U"])):
            mods[0][part]["U"][k] = torch.zeros_like(mods[0][part]["U"][k])
            if mods[0][part]["V"][k] is not None:
                mods[0][part]["V"][k] = torch.zeros_like(mods[0][part]["V"][k])
    Q = torch.randn(1, 2, 1, 4, 128, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    a, A = oracle.module_forward_general(mods, Q)
    for h in range(2):
        for net, out in (("score", a), ("target", A)):
            nt = mods[0][net]
            s = F.silu(nt["b"][-1][h].double())
            want = (nt["Wout"][h].double() @ s + nt["c"][h].double()).numpy()
            got = out[(0, h)]
            if net == "score":
                np.testing.assert_allclose(got, np.full(4, want[0]), rtol=1e-14, atol=1e-14)
            else:
                np.testing.assert_allclose(got, np.tile(want, (4, 1)), rtol=1e-14, atol=1e-14)


def test_general_module_routes_backbone_to_both_branches():
    # changing a branch moves only its own output; changing the backbone moves both
    Q = torch.randn(1, 1, 2, 3, 128, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    mods = _general(1, 1, 128, (2, 1, 2), [32], [16], [32], seed=19)
    a0, A0 = oracle.module_forward_general(mods, Q)
    mods[0]["score"]["b"][0] = mods[0]["score"]["b"][0] + 0.5
    a1, A1 = oracle.module_forward_general(mods, Q)
    assert not np.allclose(a1[(0, 0)], a0[(0, 0)]) and np.array_equal(A1[(0, 0)], A0[(0, 0)])
    mods[0]["target"]["b"][1] = mods[0]["target"]["b"][1] + 0.5
    a2, A2 = oracle.module_forward_general(mods, Q)
    assert np.array_equal(a2[(0, 0)], a1[(0, 0)]) and not np.allclose(A2[(0, 0)], A1[(0, 0)])
    mods[0]["backbone"]["b"][1] = mods[0]["backbone"]["b"][1] + 0.5
    a3, A3 = oracle.module_forward_general(mods, Q)
    assert not np.allclose(a3[(0, 0)], a2[(0, 0)]) and not np.allclose(A3[(0, 0)], A2[(0, 0)])
