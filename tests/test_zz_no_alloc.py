"""nectar_cache_attn_lse_static, the allocation-free variant of the exact
attention entry point, for callers that cannot create device buffers (a host
runtime that owns the device memory pool, plugin interfaces that pass only
inputs and outputs, latency-bound loops that cannot afford cudaMalloc).

It must give what nectar_cache_attn_lse gives, within the tolerances of the
parity tests, on consecutive calls that reuse its fixed scratch area, and it
must refuse a call whose scratch need exceeds that area.  This file is
collected last so that a run stopping at the first failure has run every
other test; it also passes on its own in a fresh process.
"""
import ctypes
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


def _inputs(L, Hkv, G, n, nq, seed):
    wl = make_workload("toy", L=L, Hkv=Hkv, G=G, n=n, nq=nq, T=1, with_local=False, with_modules=False, seed=seed)
    return wl.K.cuda(), wl.V.cuda(), wl.Q.cuda()


def _static_call(K, V, Q):
    """Call the entry point through the C ABI directly."""
    L_, Hkv, G, nq, d = Q.shape
    alpha = torch.full(Q.shape[:4], float("nan"), dtype=torch.float32, device=Q.device)
    A = torch.full(Q.shape, float("nan"), dtype=torch.float32, device=Q.device)
    st = nx.lib().nectar_cache_attn_lse_static(nx.Dims(L_, Hkv, G, d), K.data_ptr(), V.data_ptr(), K.shape[2],
                                               Q.data_ptr(), nq, ctypes.c_float(1.0 / math.sqrt(d)),
                                               alpha.data_ptr(), A.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream)
    return st, alpha, A


def _check_same(K, V, Q, alpha, A):
    """The static call runs the workspace call's plan and kernels, so the two
    must agree bit for bit; both are held to the oracle's tolerances."""
    a_ref, A_ref = nx.cache_attn_lse(K, V, Q)
    torch.cuda.synchronize()
    assert torch.equal(alpha, a_ref)
    assert torch.equal(A, A_ref)
    L_, Hkv, G, nq, d = Q.shape
    H = L_ * Hkv
    ao, Ao = oracle.cache_attn(K.reshape(H, -1, d).cpu(), V.reshape(H, -1, d).cpu(),
                               Q.reshape(H, G * nq, d).cpu(), 1.0 / math.sqrt(d))
    vmax = V.float().abs().max().item()
    assert np.abs(alpha.cpu().numpy().reshape(H, -1) - ao).max() <= ALPHA_TOL
    assert np.abs(A.cpu().numpy().reshape(H, G * nq, d) - Ao).max() <= ATT_TOL * vmax


@pytest.mark.parametrize("case", [
    [(2, 4, 2, 5000, 1, 1), (1, 3, 4, 777, 2, 2)],          # CUDA-core split kernel, twice
    [(1, 2, 4, 3000, 64, 3), (2, 2, 4, 1500, 64, 4)],       # tensor-core kernel, twice
    [(1, 2, 4, 3000, 64, 5), (3, 2, 2, 2000, 1, 6)],        # one of each, back to back
])
def test_static_matches_workspace_entry_point(case):
    for (L, Hkv, G, n, nq, seed) in case:
        K, V, Q = _inputs(L, Hkv, G, n, nq, seed)
        need = nx.cache_attn_workspace_size(L, Hkv, G, n, nq)
        assert 0 < need <= nx.static_scratch_bytes()
        st, alpha, A = _static_call(K, V, Q)
        assert st == 0, nx.lib().nectar_last_error()
        torch.cuda.synchronize()
        _check_same(K, V, Q, alpha, A)
    assert nx.device_error_flags(clear=True) == 0


def test_static_rejects_oversize():
    # 16384 (layer, KV head) pairs with 8 query rows each leave one partial per
    # head in the decode-regime kernel: 16384 * 8 * 520 B > the static area
    L, Hkv, G, n = 128, 128, 8, 64
    assert nx.cache_attn_workspace_size(L, Hkv, G, n, 1) > nx.static_scratch_bytes()
    g = torch.Generator(device="cuda").manual_seed(7)
    K = torch.randn(L, Hkv, n, 128, generator=g, device="cuda").to(torch.bfloat16)
    Q = torch.randn(L, Hkv, G, 1, 128, generator=g, device="cuda").to(torch.bfloat16)
    st, alpha, A = _static_call(K, K, Q)
    assert st == 3
    msg = nx.lib().nectar_last_error().decode()
    assert "static area holds" in msg and str(nx.static_scratch_bytes()) in msg
    torch.cuda.synchronize()
    assert torch.isnan(alpha).all()      # nothing was enqueued


def test_static_covers_tensor_core_calls():
    # the tensor-core kernel keeps at most two partials per CTA, so its scratch
    # need is bounded by the SM count whatever the shape
    for shape in [(36, 8, 4, 61440, 1024), (28, 4, 7, 131072, 64), (1, 1, 4, 128 * 300, 32)]:
        assert nx.cache_attn_workspace_size(*shape) <= nx.static_scratch_bytes()
