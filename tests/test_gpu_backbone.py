"""Module sets with a shared backbone and unequal nets (depths (D_b, D_s, D_t),
per-net widths; "Nectar", §2.4 and App. A.3) on the GPU against the oracle."""
import math

import numpy as np
import pytest
import torch

import long_context_attention_split_b200 as nx
import oracle
from nectar_inputs import make_modules_general, make_workload

MLP_TOL = 1e-2        # max |gpu - oracle| / max |oracle| per output tensor and (l, h)
ATT_TOL = 2e-3        # attention outputs: max-abs error / ||v||_inf

pytestmark = pytest.mark.gpu


def _arch_set(L, Hkv, G, depths, wb, ws, wt, seed):
    mods = make_modules_general(L, Hkv, 128, seed, "cpu", depths, wb, ws, wt)
    arch = nx.Arch(depths, wb if depths[0] else [], ws, wt)
    return mods, nx.pack_modules_arch(mods, arch, Hkv, G)


def _check_module(Q, mods, a, At):
    L, Hkv, G, nq, d = Q.shape
    ao, Ao = oracle.module_forward_general(mods, Q)
    a = a.cpu().numpy().reshape(L, Hkv, G * nq)
    At = At.cpu().numpy().reshape(L, Hkv, G * nq, d)
    for (l, h), ref in ao.items():
        ea = np.abs(a[l, h] - ref).max() / max(np.abs(ref).max(), 1e-30)
        eA = np.abs(At[l, h] - Ao[(l, h)]).max() / max(np.abs(Ao[(l, h)]).max(), 1e-30)
        assert ea <= MLP_TOL and eA <= MLP_TOL, ((l, h), ea, eA)
    return ao, Ao


CASES = [
    # (depths, width_b, width_s, width_t)
    ((2, 1, 2), [64, 48], [32, 16], [48, 96]),     # the pages' (2, 1, 2)
    ((0, 2, 3), [], [32, 208], [144, 64]),         # the pages' (0, 2, 3), unequal nets
    ((1, 3, 1), [16, 128], [48, 48], [256, 16]),   # score deeper than target
    ((3, 1, 1), [96, 64], [16, 32], [32, 16]),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("G,nq", [(2, 3), (4, 40)])
def test_module_forward_backbone(case, G, nq):
    depths, wb, ws, wt = case
    L, Hkv = 2, 2
    Q = torch.randn(L, Hkv, G, nq, 128, generator=torch.Generator().manual_seed(G * nq)).to(torch.bfloat16)
    mods, ms = _arch_set(L, Hkv, G, depths, wb, ws, wt, seed=sum(depths) + G)
    a, At = nx.module_forward(ms, Q.cuda())
    torch.cuda.synchronize()
    _check_module(Q, mods, a, At)


def test_arch_without_backbone_equals_the_classic_set():
    # D_b = 0 with equal nets is the classic set: same blob, same path, same bits
    wl = make_workload("toy", L=2, Hkv=2, G=2, n=16, nq=5, with_local=False, with_modules=True,
                       widths=[48, 32], seed=3)
    classic = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    mods = make_modules_general(2, 2, 128, 3, "cpu", (0, 2, 2), [], [48, 32], [48, 32])
    arch = nx.pack_modules_arch(mods, nx.Arch((0, 2, 2), [], [48, 32], [48, 32]), 2, 2)
    assert torch.equal(classic.blob.cpu(), arch.blob.cpu())
    Q = wl.Q.cuda()
    a0, A0 = nx.module_forward(classic, Q)
    a1, A1 = nx.module_forward(arch, Q)
    torch.cuda.synchronize()
    assert torch.equal(a0, a1) and torch.equal(A0, A1)


@pytest.mark.parametrize("case", CASES[:2])
@pytest.mark.parametrize("B,T", [(3, 40), (24, 130)])
def test_decode_backbone(case, B, T):
    depths, wb, ws, wt = case
    L, Hkv, G = 2, 2, 4
    wl = make_workload("qwen3_1p7b", L=L, Hkv=Hkv, G=G, n=16, B=B, T=T, widths=[64, 64], seed=B + T,
                       key_scale=None)
    mods, ms = _arch_set(L, Hkv, G, depths, wb, ws, wt, seed=7)
    args = tuple(t.cuda() for t in (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len))
    out = nx.decode(ms, *args)
    a, At = nx.module_forward(ms, args[0])
    torch.cuda.synchronize()
    H = L * Hkv
    ao, Ao = oracle.module_forward_general(mods, wl.Q)
    keys = [(l, h) for l in range(L) for h in range(Hkv)]
    a_o = np.stack([ao[k] for k in keys])
    A_o = np.stack([Ao[k] for k in keys])
    rows = G * wl.nq
    ref = oracle.merge_local(a_o, A_o, wl.Q.reshape(H, rows, 128), wl.q_seq, wl.q_pos,
                             wl.Kloc.reshape(H, wl.B, wl.T, 128), wl.Vloc.reshape(H, wl.B, wl.T, 128),
                             wl.local_len, 1 / math.sqrt(128))
    got = out.cpu().numpy().reshape(H, rows, 128)
    da = MLP_TOL * np.abs(a_o).max()
    dA = MLP_TOL * np.abs(A_o).max()
    vmax = max(wl.Vloc.float().abs().max().item(), np.abs(A_o).max())
    bound = da * (np.abs(A_o).max() + np.abs(ref).max()) + dA + ATT_TOL * vmax
    assert np.abs(got - ref).max() <= bound
    # the decode's fused readout merge equals module forward + merge on the GPU
    out2 = nx.merge_local(a, At, *args)
    torch.cuda.synchronize()
    assert torch.allclose(out, out2, rtol=0, atol=1e-4 * max(1.0, out2.abs().max().item()))
