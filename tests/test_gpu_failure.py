"""Failure handling on the GPU, in forms that fault, trap or hang nothing.

- The bounded waits: a wait that nothing completes gives up after its limit,
  sets bit 0 of the device error word, and the context stays usable.
- Non-finite inputs: a NaN or Inf in the document cache, the local cache or
  a query spreads only to the outputs that the definitions make depend on it
  (Eq. (3.1) for the exact attention, Eqs. (3.4)-(3.6) for the decode), every
  other output is bit for bit what the same call gives on clean inputs, no
  error bit is raised and nothing hangs.
"""
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


@pytest.fixture(autouse=True)
def _flags():
    nx.lib()
    nx.device_error_flags(clear=True)
    yield
    nx.device_error_flags(clear=True)


def test_wait_timeout_gives_up_and_the_context_survives():
    st = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    nx.check_wait_timeout(2000)           # 2 ms
    t1.record(st)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    assert 2.0 <= ms < 1000.0, ms         # it waited out its limit, then returned
    assert nx.device_error_flags(clear=True) & 1
    assert nx.device_error_flags(clear=True) == 0      # cleared
    # the next calls on the same context run and are right
    wl = make_workload("toy", L=1, Hkv=2, G=4, n=1000, nq=3, T=1, with_local=False, with_modules=False, seed=5)
    alpha, A = nx.cache_attn_lse(wl.K.cuda(), wl.V.cuda(), wl.Q.cuda())
    torch.cuda.synchronize()
    assert nx.device_error_flags(clear=True) == 0
    ao, Ao = oracle.cache_attn(wl.K, wl.V, wl.Q.reshape(1, 2, 12, 128), wl.scale)
    assert np.abs(alpha.cpu().numpy().reshape(1, 2, 12) - ao).max() <= ALPHA_TOL
    assert np.abs(A.cpu().numpy().reshape(1, 2, 12, 128) - Ao).max() <= ATT_TOL * wl.V.float().abs().max().item()


def test_wait_timeout_limit_checked_on_the_host():
    for bad in (0, -5, 1000001):
        with pytest.raises(RuntimeError, match="limit_us"):
            nx.check_wait_timeout(bad)


def _exact(K, V, Q):
    alpha, A = nx.cache_attn_lse(K, V, Q)
    torch.cuda.synchronize()
    return alpha, A


# 2 query rows per KV head: the CUDA-core split kernel; 64: the tensor-core kernel
@pytest.mark.parametrize("G,nq", [(2, 1), (4, 16)])
def test_nan_key_stays_in_its_head(G, nq):
    wl = make_workload("toy", L=2, Hkv=3, G=G, n=3000, nq=nq, T=1, with_local=False, with_modules=False, seed=G)
    K, V, Q = wl.K.cuda(), wl.V.cuda(), wl.Q.cuda()
    a0, A0 = _exact(K, V, Q)
    K[1, 2, 1234, 7] = float("nan")
    a1, A1 = _exact(K, V, Q)
    assert nx.device_error_flags(clear=True) == 0
    assert torch.isnan(a1[1, 2]).all() and torch.isnan(A1[1, 2]).all()
    keep = torch.ones(2, 3, dtype=torch.bool)
    keep[1, 2] = False
    assert torch.equal(a1[keep], a0[keep]) and torch.equal(A1[keep], A0[keep])


@pytest.mark.parametrize("G,nq", [(2, 1), (4, 16)])
def test_nan_query_stays_in_its_row(G, nq):
    wl = make_workload("toy", L=1, Hkv=2, G=G, n=2000, nq=nq, T=1, with_local=False, with_modules=False, seed=10 + G)
    K, V, Q = wl.K.cuda(), wl.V.cuda(), wl.Q.cuda()
    a0, A0 = _exact(K, V, Q)
    Q[0, 1, G - 1, nq - 1, 100] = float("nan")
    a1, A1 = _exact(K, V, Q)
    assert nx.device_error_flags(clear=True) == 0
    assert torch.isnan(a1[0, 1, G - 1, nq - 1]) and torch.isnan(A1[0, 1, G - 1, nq - 1]).all()
    keep = torch.ones(a0.shape, dtype=torch.bool, device="cuda")
    keep[0, 1, G - 1, nq - 1] = False
    assert torch.equal(a1[keep], a0[keep]) and torch.equal(A1[keep], A0[keep])


@pytest.mark.parametrize("G,nq", [(2, 1), (4, 16)])
def test_inf_value_stays_in_its_column(G, nq):
    # A = sum_j p_j v_j: an infinite v_j[c] makes column c of its head
    # infinite; alpha does not read V at all
    wl = make_workload("toy", L=1, Hkv=2, G=G, n=2000, nq=nq, T=1, with_local=False, with_modules=False, seed=20 + G)
    K, V, Q = wl.K.cuda(), wl.V.cuda(), wl.Q.cuda()
    a0, A0 = _exact(K, V, Q)
    V[0, 0, 555, 3] = float("inf")
    a1, A1 = _exact(K, V, Q)
    assert nx.device_error_flags(clear=True) == 0
    assert torch.equal(a1, a0)
    assert not torch.isfinite(A1[0, 0, ..., 3]).any()
    keep = torch.ones(A0.shape, dtype=torch.bool, device="cuda")
    keep[0, 0, ..., 3] = False
    assert torch.equal(A1[keep], A0[keep])


# 2 rows per KV head: the one-launch decode; 64 rows: local states + grouped GEMMs
@pytest.mark.parametrize("G,B", [(2, 3), (4, 16)])
def test_nan_in_local_cache_stays_in_its_sequence(G, B):
    wl = make_workload("qwen3_1p7b", seed=30 + G, key_scale=None, L=2, Hkv=2, G=G, n=16, B=B, T=40, widths=[256, 128])
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    Kl, Vl = wl.Kloc.cuda(), wl.Vloc.cuda()
    rest = (wl.q_seq.cuda(), wl.q_pos.cuda())
    Q, ll = wl.Q.cuda(), wl.local_len.cuda()
    out0 = nx.decode(mods, Q, *rest, Kl, Vl, ll)
    torch.cuda.synchronize()
    Kl[1, 0, 1, 5, 0] = float("nan")          # layer 1, KV head 0, sequence 1, local token 5
    out1 = nx.decode(mods, Q, *rest, Kl, Vl, ll)
    torch.cuda.synchronize()
    assert nx.device_error_flags(clear=True) == 0
    # decode tokens: token i is sequence i at its last position, so token 1 sees key 5
    assert torch.isnan(out1[1, 0, :, 1]).all()
    keep = torch.ones(out0.shape, dtype=torch.bool, device="cuda")
    keep[1, 0, :, 1] = False
    assert torch.equal(out1[keep], out0[keep])


@pytest.mark.parametrize("G,B", [(2, 3), (4, 16)])
def test_nan_query_stays_in_its_decode_row(G, B):
    wl = make_workload("qwen3_1p7b", seed=40 + G, key_scale=None, L=2, Hkv=2, G=G, n=16, B=B, T=40, widths=[256, 128])
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = [t.cuda() for t in (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)]
    out0 = nx.decode(mods, *args)
    torch.cuda.synchronize()
    args[0][0, 1, G - 1, 2, 9] = float("nan")   # the module and the local scores of that row
    out1 = nx.decode(mods, *args)
    torch.cuda.synchronize()
    assert nx.device_error_flags(clear=True) == 0
    assert torch.isnan(out1[0, 1, G - 1, 2]).all()
    keep = torch.ones(out0.shape, dtype=torch.bool, device="cuda")
    keep[0, 1, G - 1, 2] = False
    assert torch.equal(out1[keep], out0[keep])
