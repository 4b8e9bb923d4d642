"""GPU parity of the next rows: the Quadrature module forward (section 2.4
of the Nectar pages) and the fitting metrics (score / target MSE and the RTE
of Eq. (C.1), App. C.4), both through the C ABI, against the oracle."""
import math

import numpy as np
import pytest
import torch

import long_context_attention_split_b200 as nx
import oracle
from nectar_inputs import make_workload

pytestmark = pytest.mark.gpu

ALPHA_TOL = 1e-3
ATT_TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    nx.lib()
    nx.device_error_flags(clear=True)
    yield
    assert nx.device_error_flags(clear=True) == 0


@pytest.mark.parametrize("L,Hkv,G,n,nq,p", [
    (2, 2, 2, 700, 1, 130),     # 2 rows per KV head (split decode kernel), p over 2 tiles + 2 keys
    (2, 2, 4, 700, 9, 130),     # 36 rows (tensor-core kernel)
    (1, 3, 4, 300, 5, 1),       # p = 1: A_theta = z_1
    (1, 2, 2, 257, 64, 257),    # p = n: the module is the exact attention
])
def test_quadrature_init_and_forward(L, Hkv, G, n, nq, p):
    wl = make_workload("toy", L=L, Hkv=Hkv, G=G, n=n, nq=nq, T=1, with_local=False, with_modules=False,
                       seed=n + p)
    K, V, Q = wl.K.cuda(), wl.V.cuda(), wl.Q.cuda()
    W, Z = nx.quadrature_init(K, V, p)
    torch.cuda.synchronize()
    assert torch.equal(W.cpu(), wl.K[:, :, :p]) and torch.equal(Z.cpu(), wl.V[:, :, :p])
    a, At = nx.quadrature_forward(W, Z, Q)
    torch.cuda.synchronize()
    ao, Ao = oracle.quadrature_forward(W.cpu(), Z.cpu(), wl.Q.reshape(L, Hkv, G * nq, 128), wl.scale)
    vmax = Z.float().abs().max().item()
    assert np.abs(a.cpu().numpy().reshape(ao.shape) - ao).max() <= ALPHA_TOL
    assert np.abs(At.cpu().numpy().reshape(Ao.shape) - Ao).max() <= ATT_TOL * vmax
    if p == 1:
        assert torch.allclose(At, Z[:, :, :1].float().unsqueeze(2).expand_as(At), rtol=0, atol=1e-6)
    if p == n:
        alpha, A = nx.cache_attn_lse(K, V, Q)
        torch.cuda.synchronize()
        assert torch.equal(a, alpha) and torch.equal(At, A)


def test_quadrature_rejects_bad_p():
    wl = make_workload("toy", L=1, Hkv=1, G=1, n=64, nq=1, T=1, with_local=False, with_modules=False)
    K = wl.K.cuda()
    for p in (0, 65):
        with pytest.raises(RuntimeError, match="p ="):
            nx.quadrature_init(K, K, p)


def test_fit_metrics_against_oracle():
    # targets from the exact kernels, a module from the module kernels
    wl = make_workload("toy", L=2, Hkv=2, G=4, n=2000, nq=20, T=1, with_local=False, with_modules=True,
                       widths=[256, 128], seed=3)
    Q = wl.Q.cuda()
    alpha, A = nx.cache_attn_lse(wl.K.cuda(), wl.V.cuda(), Q)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    a, At = nx.module_forward(mods, Q)
    m = nx.fit_metrics(alpha, A, a, At, Q)
    torch.cuda.synchronize()
    rows = wl.G * wl.nq
    ref, rte = oracle.fit_metrics(alpha.cpu().reshape(-1, rows), A.cpu().reshape(-1, rows, 128),
                                  a.cpu().reshape(-1, rows), At.cpu().reshape(-1, rows, 128),
                                  wl.Q.reshape(-1, rows, 128))
    got = m.cpu().numpy().reshape(-1, 3)
    assert np.allclose(got[:, :2], ref[:, :2], rtol=1e-5, atol=0)
    assert np.abs(got[:, 2] - ref[:, 2]).max() <= 1e-5
    assert abs(got[:, 2].sum() - rte) <= 1e-4
    # a module that reproduces the targets exactly
    m0 = nx.fit_metrics(alpha, A, alpha, A, Q)
    torch.cuda.synchronize()
    assert torch.all(m0[..., :2] == 0) and torch.all(torch.isneginf(m0[..., 2]))


# ---------------------------------------------------------------------------
# the decode as a base-model attention layer: bf16, layer layout
# ---------------------------------------------------------------------------
MLP_TOL = 1e-2


def _to_layer_layout(x, wl):
    """[heads, rows, d] (rows = g * nq + i) -> [L, nq, Hkv * G, d]."""
    return x.reshape(wl.L, wl.Hkv, wl.G, wl.nq, 128).transpose(0, 3, 1, 2, 4).reshape(wl.L, wl.nq, wl.Hkv * wl.G,
                                                                                        128)


def _check_layer_out_against_oracle(wl, mods, args, got):
    """bf16 layer-layout output against the oracle, through the bf16 rounding
    (at most 2^-8 of the value, with margin): (1) the GPU's own module outputs
    through the oracle's merge, at the attention tolerance; (2) the oracle's
    module forward + merge, at the fused-decode bound."""
    a, At = nx.module_forward(mods, args[0])
    torch.cuda.synchronize()
    H = wl.heads
    loc = (wl.q_seq, wl.q_pos, wl.Kloc.reshape(H, wl.B, wl.T, 128), wl.Vloc.reshape(H, wl.B, wl.T, 128),
           wl.local_len, wl.scale)
    Qr = wl.Q.reshape(H, wl.rows, 128)
    g = got.float().cpu().numpy()
    rnd = 2.0 ** -8 * np.abs(g) * 1.01
    vloc = wl.Vloc.float().abs().max().item()
    ag = a.cpu().numpy().reshape(H, wl.rows)
    Atg = At.cpu().numpy().reshape(H, wl.rows, 128)
    ref_m = _to_layer_layout(oracle.merge_local(ag, Atg, Qr, *loc), wl)
    tol_m = ATT_TOL * max(vloc, np.abs(Atg).max())
    assert np.all(np.abs(g - ref_m) <= rnd + tol_m), np.abs(g - ref_m).max()
    ao, Ao = oracle.module_forward(wl)
    keys = [(l, h) for l in range(wl.L) for h in range(wl.Hkv)]
    a_o = np.stack([ao[k] for k in keys])
    A_o = np.stack([Ao[k] for k in keys])
    ref = oracle.merge_local(a_o, A_o, Qr, *loc)
    bound = MLP_TOL * np.abs(a_o).max() * (np.abs(A_o).max() + np.abs(ref).max()) + MLP_TOL * np.abs(A_o).max() \
        + ATT_TOL * max(vloc, np.abs(A_o).max())
    ref = _to_layer_layout(ref, wl)
    assert np.all(np.abs(g - ref) <= rnd + bound), np.abs(g - ref).max()


@pytest.mark.parametrize("kw", [
    dict(L=2, Hkv=2, G=2, n=16, B=3, T=40, widths=[256, 128]),   # 2 rows per KV head: one-launch path
    dict(L=2, Hkv=2, G=4, n=16, B=40, T=50, widths=[256, 512]),  # 160 rows: grouped-GEMM path
])
def test_decode_layer_out_is_decode_in_layer_layout(kw):
    wl = make_workload("qwen3_1p7b", seed=9, key_scale=None, **kw)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = tuple(t.cuda() for t in (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len))
    ref = nx.decode(mods, *args)                              # fp32 [L, Hkv, G, nq, d]
    got = nx.decode_layer_out(mods, *args)                    # bf16 [L, nq, Hkv*G, d]
    torch.cuda.synchronize()
    want = ref.permute(0, 3, 1, 2, 4).reshape(wl.L, wl.nq, wl.Hkv * wl.G, 128).to(torch.bfloat16)
    assert torch.equal(got, want)
    _check_layer_out_against_oracle(wl, mods, args, got)


def test_decode_layer_out_prefill_causal():
    # a prompt: 64 tokens of one sequence, token t seeing local 0..t
    wl = make_workload("toy", seed=11)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = tuple(t.cuda() for t in (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len))
    ref = nx.decode(mods, *args)
    got = nx.decode_layer_out(mods, *args)
    torch.cuda.synchronize()
    want = ref.permute(0, 3, 1, 2, 4).reshape(wl.L, wl.nq, wl.Hkv * wl.G, 128).to(torch.bfloat16)
    assert torch.equal(got, want)
    _check_layer_out_against_oracle(wl, mods, args, got)


def test_decode_layer_out_prompt_several_sequences():
    # prompts of 3 sequences at once (64 tokens of each, token t at local
    # position t), the bf16 layer layout against the oracle
    T = 64
    B = 3
    nq = B * T
    q_seq = [b for b in range(B) for _ in range(T)]
    q_pos = [t for _ in range(B) for t in range(T)]
    wl = make_workload("toy", seed=12, L=2, Hkv=2, G=2, n=16, B=B, T=T, nq=nq, widths=[256, 128],
                       q_seq=q_seq, q_pos=q_pos, local_len=[T, T - 5, 40])
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = tuple(t.cuda() for t in (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len))
    got = nx.decode_layer_out(mods, *args)
    torch.cuda.synchronize()
    assert nx.device_error_flags() == 0
    _check_layer_out_against_oracle(wl, mods, args, got)
