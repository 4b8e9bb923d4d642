"""Parity at the full sizes of the workloads, in the launch configuration
bench.py times: every (l, h) runs on the GPU, and sampled heads and tokens
are recomputed by the oracle one by one."""
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
MLP_TOL = 1e-2


def sample_heads(wl, k, seed):
    rng = np.random.default_rng(seed)
    hs = {(0, 0), (wl.L - 1, wl.Hkv - 1)}
    while len(hs) < k:
        hs.add((int(rng.integers(wl.L)), int(rng.integers(wl.Hkv))))
    return sorted(hs)


def check_exact(wl, alpha, A, heads, tokens):
    """(alpha, A) of the rows of `tokens` (all G query heads) against the oracle."""
    for (l, h) in heads:
        X = wl.Q[l, h][:, tokens].reshape(1, -1, 128).cpu()
        ao, Ao = oracle.cache_attn(wl.K[l, h][None].cpu(), wl.V[l, h][None].cpu(), X, wl.scale)
        ag = alpha[l, h][:, tokens].reshape(1, -1).cpu().numpy()
        Ag = A[l, h][:, tokens].reshape(1, -1, 128).cpu().numpy()
        vmax = wl.V[l, h].float().abs().max().item()
        assert np.abs(ag - ao).max() <= ALPHA_TOL, ((l, h), np.abs(ag - ao).max())
        assert np.abs(Ag - Ao).max() <= ATT_TOL * vmax, ((l, h), np.abs(Ag - Ao).max())


def readout_scale(wl, l, h, net, X):
    """Scale of a net's outputs for the relative MLP tolerance when a (l, h)
    has only a few query rows: the largest root-sum-square of the readout's
    terms, max over rows and outputs j of sqrt(sum_i (W[j, i] h_i)^2) + |c_j|,
    with h the oracle's last hidden state (the oracle's chain of the net's
    hidden layers with an identity readout).  A sum of independently rounded
    terms errs on that scale, while its value can cancel towards 0."""
    nd = wl.modules[l][net]
    H = wl.widths[l]
    ident = dict(nd, Wout=torch.eye(H, dtype=torch.bfloat16).expand(wl.Hkv, H, H),
                 c=torch.zeros(wl.Hkv, H, dtype=torch.bfloat16))
    params, widths = oracle.flatten_chain(None, ident, [h])
    hid = oracle.chain(params, X, widths, H)[0]                   # [rows, H], fp64
    W = nd["Wout"][h].double().cpu().numpy()                       # [dout, H]
    c = nd["c"][h].double().cpu().numpy()                          # [dout]
    rss = np.sqrt(((hid[:, None, :] * W[None, :, :]) ** 2).sum(-1))   # [rows, dout]
    return float((rss + np.abs(c)[None, :]).max())


def check_decode(wl, out, heads, tokens, a_gpu=None, At_gpu=None):
    """Fused decode output of the rows of `tokens` against the oracle's
    module forward + merge for those rows.  With the GPU's own module
    outputs (a_gpu, At_gpu from nx.module_forward) the merge step is also
    checked alone, at the attention tolerance: those outputs through the
    oracle's merge (Eqs. (3.4)-(3.5)) must give the decode's out."""
    tok = torch.as_tensor(tokens)
    for (l, h) in heads:
        H = wl.widths[l]
        X = wl.Q[l, h][:, tok].reshape(1, -1, 128).cpu()
        a = oracle.mlp(oracle.flatten_net(wl.modules[l]["score"], [h]), X, wl.depth, H, 1)[..., 0]
        At = oracle.mlp(oracle.flatten_net(wl.modules[l]["target"], [h]), X, wl.depth, H, 128)
        loc = (wl.q_seq[tok].cpu(), wl.q_pos[tok].cpu(), wl.Kloc[l, h][None].cpu(), wl.Vloc[l, h][None].cpu(),
               wl.local_len.cpu())
        ref = oracle.merge_local(a, At, X, *loc, wl.scale)
        got = out[l, h][:, tok].reshape(1, -1, 128).cpu().numpy()
        vloc = wl.Vloc[l, h].float().abs().max().item()
        vmax = max(vloc, np.abs(At).max())
        bound = MLP_TOL * np.abs(a).max() * (np.abs(At).max() + np.abs(ref).max()) + MLP_TOL * np.abs(At).max() \
            + ATT_TOL * vmax
        err = np.abs(got - ref).max()
        assert err <= bound, ((l, h), err, bound)
        if a_gpu is not None:
            ag = a_gpu[l, h][:, tok].reshape(1, -1).cpu().numpy()
            Atg = At_gpu[l, h][:, tok].reshape(1, -1, 128).cpu().numpy()
            # the module outputs themselves, at the MLP tolerance relative to
            # the readout's term scale (with 2 rows per (l, h) max|a| itself
            # can be near 0 when the readout's terms cancel)
            sa = readout_scale(wl, l, h, "score", X)
            st = readout_scale(wl, l, h, "target", X)
            assert np.abs(ag - a).max() <= MLP_TOL * sa, ((l, h), np.abs(ag - a).max(), sa)
            assert np.abs(Atg - At).max() <= MLP_TOL * st, ((l, h), np.abs(Atg - At).max(), st)
            ref_m = oracle.merge_local(ag, Atg, X, *loc, wl.scale)
            tol_m = ATT_TOL * max(vloc, np.abs(Atg).max())
            err_m = np.abs(got - ref_m).max()
            assert err_m <= tol_m, ((l, h), err_m, tol_m)


def test_qwen3_1p7b_decode_full():
    """The headline step exactly as bench.py runs it: 28 x 8 KV heads, G = 2,
    n = 32768 with per-head key scales, H = 512, one decode token after 512
    local tokens (the one-launch decode with its local CTAs first, and the
    split exact-attention kernel at 2 rows per KV head).  Every (l, h) is
    checked: exact (alpha, A), the module outputs, the merge step alone and
    the decode output."""
    wl = make_workload("qwen3_1p7b", device="cuda")
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G, device="cuda")
    alpha, A = nx.cache_attn_lse(wl.K, wl.V, wl.Q)
    out = nx.decode(mods, wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
    a, At = nx.module_forward(mods, wl.Q)
    torch.cuda.synchronize()
    assert nx.device_error_flags() == 0
    heads = [(l, h) for l in range(wl.L) for h in range(wl.Hkv)]
    check_exact(wl, alpha, A, heads, [0])
    check_decode(wl, out, heads, [0], a, At)
    del wl, mods, alpha, A, out, a, At
    torch.cuda.empty_cache()


def test_qwen3_4b_targets_full():
    """36 x 8 heads, n = 61440 with heavy hitters, 4096 query rows per head."""
    wl = make_workload("qwen3_4b_targets", device="cuda")
    alpha, A = nx.cache_attn_lse(wl.K, wl.V, wl.Q)
    torch.cuda.synchronize()
    assert nx.device_error_flags() == 0
    check_exact(wl, alpha, A, sample_heads(wl, 3, 1), [0, 511, 1023])
    del wl, alpha, A
    torch.cuda.empty_cache()


def test_qwen25_7b_decode_full():
    """28 x 4 heads, G = 7, n = 131072, 64 sequences x 256 local tokens, H = 768."""
    wl = make_workload("qwen25_7b_decode", device="cuda")
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G, device="cuda")
    alpha, A = nx.cache_attn_lse(wl.K, wl.V, wl.Q)
    out = nx.decode(mods, wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
    full = nx.merge_local(alpha, A, wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
    a, At = nx.module_forward(mods, wl.Q)
    torch.cuda.synchronize()
    assert nx.device_error_flags() == 0
    heads = sample_heads(wl, 3, 2)
    check_exact(wl, alpha, A, heads, [0, 37, 63])
    check_decode(wl, out, heads, [0, 37, 63], a, At)
    # Eq. (3.4): merging the exact (alpha, A) is full attention over document + local
    (l, h) = heads[0]
    tok = torch.tensor([5])
    ref = oracle.full_attention(wl.K[l, h][None].cpu(), wl.V[l, h][None].cpu(),
                                wl.Q[l, h][:, tok].reshape(1, -1, 128).cpu(), wl.q_seq[tok].cpu(),
                                wl.q_pos[tok].cpu(), wl.Kloc[l, h][None].cpu(), wl.Vloc[l, h][None].cpu(),
                                wl.local_len.cpu(), wl.scale)
    got = full[l, h][:, tok].reshape(1, -1, 128).cpu().numpy()
    vmax = max(wl.V[l, h].float().abs().max().item(), wl.Vloc[l, h].float().abs().max().item())
    assert np.abs(got - ref).max() <= ATT_TOL * vmax
    del wl, mods, alpha, A, out, full, a, At
    torch.cuda.empty_cache()


def test_qwen25_7b_decode_rho10_full():
    """The Qwen2.5-7B-shaped decode at the stated capacity rho = 10 %: H = 1152
    (10.12 % of 2nd per (l, h); H = 768 is 4.99 %), 28 x 4 heads, G = 7,
    n = 131072, 64 sequences x 256 local tokens."""
    wl = make_workload("qwen25_7b_decode", device="cuda", H=1152)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G, device="cuda")
    out = nx.decode(mods, wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
    a, At = nx.module_forward(mods, wl.Q)
    torch.cuda.synchronize()
    assert nx.device_error_flags() == 0
    check_decode(wl, out, sample_heads(wl, 3, 3), [0, 31, 63], a, At)
    del wl, mods, out, a, At
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,rho", [(1, 0.10), (16, 0.10), (256, 0.10), (16, 0.01), (16, 0.05)])
def test_llama8b_sweep_full(B, rho):
    """32 x 8 heads, G = 4, n = 65536, 128 local tokens, non-uniform widths."""
    wl = make_workload("llama8b_sweep", device="cuda", B=B, rho=rho)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G, device="cuda")
    alpha, A = nx.cache_attn_lse(wl.K, wl.V, wl.Q)
    out = nx.decode(mods, wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
    a, At = nx.module_forward(mods, wl.Q)
    torch.cuda.synchronize()
    assert nx.device_error_flags() == 0
    heads = sample_heads(wl, 3, B)
    tokens = sorted({0, B // 2, B - 1})
    check_exact(wl, alpha, A, heads, tokens)
    check_decode(wl, out, heads, tokens, a, At)
    del wl, mods, alpha, A, out, a, At
    torch.cuda.empty_cache()
