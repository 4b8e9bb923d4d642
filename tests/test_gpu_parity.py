"""GPU parity: every entry point of libnectar.so against the CPU oracle on the
same seeded inputs.

Tolerances (the method's acceptance bar; the fused-decode bound is derived
from the MLP and attention tolerances below):
  alpha            |gpu - oracle| <= 1e-3 absolute
  A, merged out    max|gpu - oracle| <= 2e-3 * ||v||_inf  (v: the values involved)
  MLP outputs      max|gpu - oracle| / max|oracle| <= 1e-2 per (l, h) and tensor
  fused decode     the merge of outputs carrying the MLP tolerance (bound below)
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
MLP_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    nx.lib()
    nx.device_error_flags(clear=True)
    yield
    assert nx.device_error_flags(clear=True) == 0


def cuda(t):
    return None if t is None else t.cuda()


def check_attn(alpha_g, A_g, alpha_o, A_o, vmax, what=""):
    da = np.abs(alpha_g - alpha_o).max() if alpha_o.size else 0.0
    dA = np.abs(A_g - A_o).max() if A_o.size else 0.0
    assert da <= ALPHA_TOL, f"{what} alpha err {da}"
    assert dA <= ATT_TOL * vmax, f"{what} A err {dA} > {ATT_TOL} * {vmax}"


def run_cache_attn(L, Hkv, G, n, nq, seed=0, key_scale=None):
    wl = make_workload("toy", L=L, Hkv=Hkv, G=G, n=n, nq=nq, T=1, with_local=False, with_modules=False,
                       seed=seed, key_scale=key_scale)
    alpha, A = nx.cache_attn_lse(cuda(wl.K), cuda(wl.V), cuda(wl.Q))
    torch.cuda.synchronize()
    ao, Ao = oracle.cache_attn(wl.K, wl.V, wl.Q.reshape(L, Hkv, G * nq, 128), wl.scale)
    return wl, alpha.cpu().numpy().reshape(L, Hkv, G * nq), A.cpu().numpy().reshape(L, Hkv, G * nq, 128), ao, Ao


# ---------------------------------------------------------------------------
# (i) exact cached-token attention
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L,Hkv,G,n,nq", [
    (1, 1, 4, 4096, 64),      # toy: 256 rows, 64 tiles
    (1, 3, 2, 1000, 1),       # ragged tail (1000 = 15*64 + 40), R = 2
    (2, 2, 1, 129, 1),        # R = 1, one key past a tile
    (1, 2, 4, 700, 1),        # R = 4
    (1, 2, 7, 333, 1),        # R = 7 (16-lane groups)
    (2, 1, 8, 64, 1),         # R = 8, exactly one tile
    (1, 1, 3, 1, 1),          # n = 1
    (3, 2, 2, 5000, 3),       # 6 rows, several heads per CTA range
    # tensor-core path (more than 8 query rows per KV head)
    (1, 1, 3, 777, 3),        # 9 rows: one partial 128-row tile, ragged keys
    (1, 2, 2, 1000, 65),      # 130 rows: two row tiles, the second with 2 rows
    (4, 8, 4, 1000, 4),       # 16 rows, 32 heads: units cut between CTAs
    (1, 2, 8, 128, 128),      # 1024 rows, n = one key tile: units whole in a CTA
    (1, 1, 4, 100, 32),       # n < one key tile
    (2, 2, 4, 8192, 128),     # 512 rows x 64 key tiles
    # one query tile per unit: the key range split between the warpgroups
    (1, 2, 4, 266, 16),       # 64 rows, 5 key tiles: halves of 3 and 2, ragged last tile
    (2, 8, 4, 3000, 16),      # 64 rows, 16 heads: units cut into short segments between CTAs
    (1, 1, 2, 64 * 2, 40),    # 80 rows, exactly two key tiles: one each
    (256, 1, 2, 200, 1),      # 256 layers (NECTAR_MAX_LAYERS)
    # one head cut over every CTA: more partials per head than a warp has lanes
    (1, 1, 2, 65536, 1),      # 1024 key tiles over all CTAs
    (1, 1, 1, 1900, 1),       # ~30 one-tile partials
])
def test_cache_attn_parity(L, Hkv, G, n, nq):
    wl, ag, Ag, ao, Ao = run_cache_attn(L, Hkv, G, n, nq, seed=n + G)
    check_attn(ag, Ag, ao, Ao, wl.V.float().abs().max().item(), f"n={n}")


# The tensor-core kernel's lockstep rest: after the whole rounds, each
# remaining unit (two or more query units per head) in S equal key parts,
# item p * U + u on CTA item % C.  On 148 SMs: 4 heads x 2 query units, 148
# key tiles -> no whole round, S = 37, two items on every CTA (both partial
# slots); 75 heads x 2 query units, 37 key tiles -> one whole round, then 2
# units in 37 one-tile parts.
@pytest.mark.parametrize("L,Hkv,G,n,nq", [
    (1, 4, 4, 148 * 64, 128),
    (1, 75, 2, 37 * 64, 129),
])
def test_cache_attn_tc_lockstep_rest(L, Hkv, G, n, nq):
    wl, ag, Ag, ao, Ao = run_cache_attn(L, Hkv, G, n, nq, seed=n + Hkv)
    check_attn(ag, Ag, ao, Ao, wl.V.float().abs().max().item(), f"lockstep n={n}")


# 3-16 query rows per KV head: the transposed tensor-core split kernel
# (keys on the TMEM lanes).  Cases: a ragged single tile, many short heads per
# CTA range (each CTA crosses 4 heads: the double-buffered Q and O^T are
# reused), a head cut over several CTAs, 16 rows, and the same shapes on the
# CUDA-core kernel (NECTAR_TCT=0) for comparison.
@pytest.mark.parametrize("L,Hkv,G,n,nq", [
    (1, 2, 3, 100, 1),        # 3 rows, n < one 128-key tile
    (30, 20, 4, 100, 1),      # 600 one-tile heads: ~4 head ranges per CTA
    (2, 4, 5, 20000, 1),      # 5 rows, each head cut over ~18 CTAs
    (1, 3, 8, 1537, 2),       # 16 rows, ragged tail of 1 key
    (2, 2, 2, 5000, 6),       # 12 rows (QC = 16)
    (1, 2, 4, 5000, 5),       # 20 rows: 32 query columns
    (2, 3, 4, 3000, 16),      # 64 rows: 64 query columns, heads cut over CTAs
    (1, 2, 8, 1000, 6),       # 48 rows, ragged tail
    (1, 1, 5, 131072, 1),     # 5 rows, one head cut over every CTA
])
def test_cache_attn_tct(L, Hkv, G, n, nq, monkeypatch):
    wl, ag, Ag, ao, Ao = run_cache_attn(L, Hkv, G, n, nq, seed=n + 7 * G)
    vmax = wl.V.float().abs().max().item()
    check_attn(ag, Ag, ao, Ao, vmax, f"tct n={n}")
    if G * nq <= 8:
        monkeypatch.setenv("NECTAR_TCT", "0")
        _, ag0, Ag0, _, _ = run_cache_attn(L, Hkv, G, n, nq, seed=n + 7 * G)
        check_attn(ag0, Ag0, ao, Ao, vmax, f"split n={n}")
        assert np.abs(ag - ag0).max() <= ALPHA_TOL and np.abs(Ag - Ag0).max() <= ATT_TOL * vmax


# 33-64 query rows per KV head: the tensor-core kernel with the rows of the
# query tile repeated, each row's keys of a tile halved between two
# threads, and the two halves joined at the end.  Cases: both halves of the
# last tile partly valid, the second half of the last tile empty, one key
# tile (one warpgroup, no key split), n < 32 (the second half never holds a
# key), heads cut over CTAs (partials); each also with NECTAR_TC_DUP=0.
@pytest.mark.parametrize("L,Hkv,G,n,nq", [
    (1, 2, 3, 700, 11),       # 33 rows, last tile 60 keys
    (1, 3, 4, 650, 16),       # 64 rows, last tile 10 keys
    (2, 2, 7, 64, 9),         # 63 rows, exactly one key tile
    (1, 1, 8, 40, 8),         # 64 rows, n = 40
    (3, 4, 4, 20000, 16),     # 64 rows, heads cut over CTAs
])
def test_cache_attn_tc_repeated_rows(L, Hkv, G, n, nq, monkeypatch):
    wl, ag, Ag, ao, Ao = run_cache_attn(L, Hkv, G, n, nq, seed=n + 11 * G)
    vmax = wl.V.float().abs().max().item()
    check_attn(ag, Ag, ao, Ao, vmax, f"repeated rows n={n}")
    monkeypatch.setenv("NECTAR_TC_DUP", "0")
    _, ag0, Ag0, _, _ = run_cache_attn(L, Hkv, G, n, nq, seed=n + 11 * G)
    check_attn(ag0, Ag0, ao, Ao, vmax, f"one thread per row n={n}")
    assert np.abs(ag - ag0).max() <= ALPHA_TOL and np.abs(Ag - Ag0).max() <= ATT_TOL * vmax


@pytest.mark.parametrize("G,nq", [(5, 1), (4, 16)])
def test_cache_attn_tct_repeatable(G, nq):
    # a head spread over several CTAs with several tiles each: ten calls give
    # the same bits (the partials are summed in a fixed order; a call that
    # read a head's O^T before its last tiles had landed would not)
    wl = make_workload("toy", L=2, Hkv=4, G=G, n=20000, nq=nq, T=1, with_local=False, with_modules=False, seed=3)
    K, V, Q = wl.K.cuda(), wl.V.cuda(), wl.Q.cuda()
    a0, A0 = nx.cache_attn_lse(K, V, Q)
    for _ in range(9):
        a1, A1 = nx.cache_attn_lse(K, V, Q)
        torch.cuda.synchronize()
        assert torch.equal(a1, a0) and torch.equal(A1, A0)
    ao, Ao = oracle.cache_attn(wl.K, wl.V, wl.Q.reshape(2, 4, G * nq, 128), wl.scale)
    check_attn(a0.cpu().numpy().reshape(ao.shape), A0.cpu().numpy().reshape(Ao.shape), ao, Ao,
               wl.V.float().abs().max().item(), "tct repeat")


@pytest.mark.parametrize("nq", [1, 12])
def test_cache_attn_tct_running_max_moves(nq):
    # 4 or 48 rows: after 40 tiles of ordinary scores a key scores ~ +10
    # (natural log units) higher for two of the rows, so the running maximum
    # of those rows moves past the 2^8 slack and their O^T columns are
    # rescaled in TMEM
    L, Hkv, G, n = 1, 2, 4, 9000
    g = torch.Generator().manual_seed(21)
    K = torch.randn(L, Hkv, n, 128, generator=g)
    V = torch.randn(L, Hkv, n, 128, generator=g)
    Q = torch.randn(L, Hkv, G, nq, 128, generator=g)
    u = Q[0, 1, 1, 0] / Q[0, 1, 1, 0].norm()
    K[0, 1, 5123] = 40.0 * u
    w = Q[0, 0, 3, 0] / Q[0, 0, 3, 0].norm()
    K[0, 0, 8999] = 45.0 * w             # the very last key of a head
    K, V, Q = K.to(torch.bfloat16), V.to(torch.bfloat16), Q.to(torch.bfloat16)
    alpha, A = nx.cache_attn_lse(cuda(K), cuda(V), cuda(Q))
    torch.cuda.synchronize()
    ao, Ao = oracle.cache_attn(K, V, Q.reshape(L, Hkv, G * nq, 128), 1 / math.sqrt(128))
    check_attn(alpha.cpu().numpy().reshape(ao.shape), A.cpu().numpy().reshape(Ao.shape), ao, Ao,
               V.float().abs().max().item(), "tct rescale")


def test_cache_attn_key_scale_and_heavy_hitters():
    wl, ag, Ag, ao, Ao = run_cache_attn(2, 2, 2, 3000, 2, seed=5, key_scale=(0.5, 2.0))
    check_attn(ag, Ag, ao, Ao, wl.V.float().abs().max().item())
    wl = make_workload("qwen3_4b_targets", L=1, Hkv=2, n=2048, nq=16, seed=9)
    alpha, A = nx.cache_attn_lse(cuda(wl.K), cuda(wl.V), cuda(wl.Q))
    ao, Ao = oracle.cache_attn(wl.K, wl.V, wl.Q.reshape(1, 2, wl.rows, 128), wl.scale)
    check_attn(alpha.cpu().numpy().reshape(ao.shape), A.cpu().numpy().reshape(Ao.shape), ao, Ao,
               wl.V.float().abs().max().item(), "heavy")


def test_cache_attn_empty_document():
    Q = torch.randn(1, 2, 2, 3, 128).to(torch.bfloat16).cuda()
    K = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16).cuda()
    alpha, A = nx.cache_attn_lse(K, K, Q)
    assert torch.all(torch.isneginf(alpha)) and torch.all(A == 0)


def test_cache_attn_invariants_on_gpu():
    wl, ag, Ag, _, _ = run_cache_attn(1, 2, 4, 2048, 2, seed=77)
    S = torch.einsum("hrd,hnd->hrn", wl.Q.reshape(2, 8, 128).double(), wl.K[0].double()) * wl.scale
    smax = S.max(-1).values.numpy()
    assert np.all(ag[0] >= smax - ALPHA_TOL) and np.all(ag[0] <= smax + math.log(2048) + ALPHA_TOL)
    vmin = wl.V[0].double().amin(1).numpy()[:, None, :]
    vmax = wl.V[0].double().amax(1).numpy()[:, None, :]
    assert np.all(Ag[0] >= vmin - 1e-5) and np.all(Ag[0] <= vmax + 1e-5)


def test_cache_attn_workspace_errors():
    wl = make_workload("toy", L=1, Hkv=1, G=2, n=256, nq=1, with_local=False, with_modules=False)
    ws = nx.cache_attn_workspace_size(1, 1, 2, 256, 1)
    assert ws > 0
    small = torch.empty(ws - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(nx.NectarError) as e:
        nx.cache_attn_lse(cuda(wl.K), cuda(wl.V), cuda(wl.Q), workspace=small)
    assert e.value.status == 3


def test_cache_attn_tc_heavy_hitters_config3_shape():
    """Regression-target shape (4096 query rows per head) on a reduced cache:
    heavy-hitter keys with a +6 logit, tensor-core path."""
    wl = make_workload("qwen3_4b_targets", L=1, Hkv=2, n=4096, nq=1024, seed=11)
    alpha, A = nx.cache_attn_lse(cuda(wl.K), cuda(wl.V), cuda(wl.Q))
    torch.cuda.synchronize()
    sel = torch.arange(0, wl.rows, 37)      # sampled rows, recomputed by the oracle
    for h in range(2):
        ao, Ao = oracle.cache_attn(wl.K[0, h][None], wl.V[0, h][None], wl.Q[0, h].reshape(1, -1, 128)[:, sel],
                                   wl.scale)
        check_attn(alpha[0, h].reshape(1, -1)[:, sel].cpu().numpy(),
                   A[0, h].reshape(1, -1, 128)[:, sel].cpu().numpy(), ao, Ao, wl.V.float().abs().max().item())


@pytest.mark.parametrize("nq", [64, 16])
def test_cache_attn_tc_running_max_moves(nq):
    """A key deep in the cache that scores far above everything before it, for
    half of the query rows only: the running maximum moves by more than 2^8
    inside a unit for some rows of a warp and not for others.  nq = 16 gives
    64 rows per KV head, one query tile: the two softmax warpgroups take the
    two halves of the keys, and the spike falls inside the second half."""
    g = torch.Generator().manual_seed(21)
    L, Hkv, G, n = 2, 2, 4, 3000
    K = torch.randn(L, Hkv, n, 128, generator=g)
    V = torch.randn(L, Hkv, n, 128, generator=g).to(torch.bfloat16)
    Q = torch.randn(L, Hkv, G, nq, 128, generator=g)
    u = torch.nn.functional.normalize(torch.randn(128, generator=g), dim=0)
    Q[..., ::2, :] += 3.0 * u           # every other token of every query head
    K[:, :, 2345] = 40.0 * u            # scores ~ +10 (natural log units) for those rows
    K, Q = K.to(torch.bfloat16), Q.to(torch.bfloat16)
    alpha, A = nx.cache_attn_lse(cuda(K), cuda(V), cuda(Q))
    torch.cuda.synchronize()
    ao, Ao = oracle.cache_attn(K, V, Q.reshape(L, Hkv, G * nq, 128), 1 / math.sqrt(128))
    check_attn(alpha.cpu().numpy().reshape(ao.shape), A.cpu().numpy().reshape(Ao.shape), ao, Ao,
               V.float().abs().max().item(), "rescale")


def test_cache_attn_full_size_sampled():
    """Qwen3-1.7B shape at full n = 32768, every head on the GPU; sampled
    heads (first, last, and two seeded ones) recomputed by the oracle."""
    wl = make_workload("qwen3_1p7b", device="cuda", with_local=False, with_modules=False)
    alpha, A = nx.cache_attn_lse(wl.K, wl.V, wl.Q)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    heads = [(0, 0), (wl.L - 1, wl.Hkv - 1)] + [tuple(x) for x in rng.integers(0, [wl.L, wl.Hkv], (2, 2))]
    for (l, h) in heads:
        ao, Ao = oracle.cache_attn(wl.K[l, h][None], wl.V[l, h][None], wl.Q[l, h].reshape(1, wl.rows, 128), wl.scale)
        check_attn(alpha[l, h].reshape(1, -1).cpu().numpy(), A[l, h].reshape(1, wl.rows, 128).cpu().numpy(), ao, Ao,
                   wl.V[l, h].float().abs().max().item(), f"head {(l, h)}")


# ---------------------------------------------------------------------------
# (iii) merge with exact local attention
# ---------------------------------------------------------------------------
def merge_case(G, nq, B, T, q_seq, q_pos, local_len, L=1, Hkv=2, seed=0):
    g = torch.Generator().manual_seed(seed)
    rows = G * nq
    Q = torch.randn(L, Hkv, G, nq, 128, generator=g).to(torch.bfloat16)
    Kl = torch.randn(L, Hkv, B, T, 128, generator=g).to(torch.bfloat16)
    Vl = torch.randn(L, Hkv, B, T, 128, generator=g).to(torch.bfloat16)
    a = (torch.randn(L, Hkv, G, nq, generator=g) * 2).float()
    Ad = torch.randn(L, Hkv, G, nq, 128, generator=g).float()
    qs = torch.tensor(q_seq, dtype=torch.int32)
    qp = torch.tensor(q_pos, dtype=torch.int32)
    ll = torch.tensor(local_len, dtype=torch.int32)
    out = nx.merge_local(cuda(a), cuda(Ad), cuda(Q), cuda(qs), cuda(qp), cuda(Kl), cuda(Vl), cuda(ll))
    torch.cuda.synchronize()
    H = L * Hkv
    ref = oracle.merge_local(a.reshape(H, rows), Ad.reshape(H, rows, 128), Q.reshape(H, rows, 128), qs, qp,
                             Kl.reshape(H, B, T, 128), Vl.reshape(H, B, T, 128), ll, 1 / math.sqrt(128))
    vmax = max(Vl.float().abs().max().item(), Ad.abs().max().item())
    err = np.abs(out.cpu().numpy().reshape(H, rows, 128) - ref).max()
    assert err <= ATT_TOL * vmax, err
    return out, Ad


@pytest.mark.parametrize("G", [1, 2, 4, 7, 8, 11])
def test_merge_decode_shapes(G):
    B, T = 3, 70
    merge_case(G, B, B, T, list(range(B)), [T - 1] * B, [T, 41, 1], seed=G)


def test_merge_prefill_causal():
    T = 64
    merge_case(4, T, 1, T, [0] * T, list(range(T)), [T], L=1, Hkv=1, seed=3)


def test_merge_edge_cases():
    # q_pos 0; local_len 1; local_len = T_max; local_len 0 -> out = A_doc;
    # q_pos past local_len (sees local_len tokens); q_pos = INT32_MAX (sees
    # all local_len tokens: the visible count q_pos + 1 must not wrap)
    T = 9
    out, Ad = merge_case(3, 6, 4, T, [0, 1, 2, 3, 1, 2], [0, 5, T - 1, 2, 8, 2**31 - 1], [T, 1, T, 0], seed=4)
    o = out.cpu().reshape(2, 3, 6, 128)
    A = Ad.reshape(2, 3, 6, 128)
    assert torch.equal(o[:, :, 3], A[:, :, 3])
    # the INT32_MAX token and a token at the last position see the same keys
    out2, _ = merge_case(3, 6, 4, T, [0, 1, 2, 3, 1, 2], [0, 5, T - 1, 2, 8, T - 1], [T, 1, T, 0], seed=4)
    assert torch.equal(out[..., 5, :], out2[..., 5, :])


def test_merge_bad_metadata_flags():
    nx.device_error_flags(clear=True)
    out, Ad = merge_case(2, 2, 2, 4, [0, 1], [3, 3], [4, 4], seed=5)
    assert nx.device_error_flags(clear=True) == 0
    g = torch.Generator().manual_seed(1)
    Q = torch.randn(1, 1, 2, 2, 128, generator=g).to(torch.bfloat16).cuda()
    Kl = torch.randn(1, 1, 2, 4, 128, generator=g).to(torch.bfloat16).cuda()
    a = torch.zeros(1, 1, 2, 2).cuda()
    Ad = torch.randn(1, 1, 2, 2, 128).cuda()
    qs = torch.tensor([0, 5], dtype=torch.int32).cuda()      # 5 is not a sequence
    qp = torch.tensor([3, 3], dtype=torch.int32).cuda()
    ll = torch.tensor([4, 9], dtype=torch.int32).cuda()       # 9 > T_max
    out = nx.merge_local(a, Ad, Q, qs, qp, Kl, Kl, ll)
    flags = nx.device_error_flags(clear=True)
    assert flags & 2
    assert torch.equal(out[..., 1, :], Ad[..., 1, :])


# many query rows per KV head: the tensor-core local kernels (one job per
# (KV head, token), 128-key tiles).  G <= 16 with at most 512 local tokens
# runs the transposed kernel (keys on the TMEM lanes), G = 33 the kernel with
# the query heads on the lanes, T = 600 the warp kernel.
@pytest.mark.parametrize("G,T", [(1, 300), (4, 33), (7, 256), (9, 200), (16, 512), (33, 130), (4, 600)])
def test_merge_many_tokens(G, T):
    nq = max(128 // G + 1, 8)
    B = 5
    g = torch.Generator().manual_seed(G * 1000 + T)
    q_seq = torch.randint(0, B, (nq,), generator=g).tolist()
    local_len = [T, 0, 1, T // 2 + 3, T - 1]
    q_pos = torch.randint(0, T, (nq,), generator=g).tolist()
    q_pos[0] = 0
    q_pos[1] = 2**31 - 1          # sees its whole sequence
    out, Ad = merge_case(G, nq, B, T, q_seq, q_pos, local_len, seed=G + T)
    # tokens of the sequence with no local tokens keep the document term
    o = out.cpu().reshape(2, G, nq, 128)
    A = Ad.reshape(2, G, nq, 128)
    for i, b in enumerate(q_seq):
        if b == 1:
            assert torch.equal(o[:, :, i], A[:, :, i])


@pytest.mark.parametrize("G,T", [(4, 33), (7, 256), (16, 130)])
def test_merge_many_tokens_without_transposed_kernel(G, T, monkeypatch):
    # the warp kernel (G <= 8) and the row-per-head tensor-core kernel (G > 8)
    monkeypatch.setenv("NECTAR_LOCAL_TCT", "0")
    test_merge_many_tokens(G, T)


def test_merge_prefill_causal_many_tiles():
    T = 300
    merge_case(4, T, 1, T, [0] * T, list(range(T)), [T], L=1, Hkv=1, seed=13)


def test_merge_tc_running_max_moves():
    # keys of the second 128-key tile score far above the first: the running
    # maximum jumps by more than the lazy-rescale slack inside one job
    G, nq, B, T = 4, 40, 2, 256
    g = torch.Generator().manual_seed(21)
    rows = G * nq
    Q = torch.randn(1, 2, G, nq, 128, generator=g).to(torch.bfloat16)
    Kl = torch.randn(1, 2, B, T, 128, generator=g)
    Kl[:, :, :, 128:] *= 8.0
    Kl = Kl.to(torch.bfloat16)
    Vl = torch.randn(1, 2, B, T, 128, generator=g).to(torch.bfloat16)
    a = torch.randn(1, 2, G, nq, generator=g).float()
    Ad = torch.randn(1, 2, G, nq, 128, generator=g).float()
    qs = torch.tensor([i % B for i in range(nq)], dtype=torch.int32)
    qp = torch.full((nq,), T - 1, dtype=torch.int32)
    ll = torch.tensor([T, T], dtype=torch.int32)
    out = nx.merge_local(cuda(a), cuda(Ad), cuda(Q), cuda(qs), cuda(qp), cuda(Kl), cuda(Vl), cuda(ll))
    torch.cuda.synchronize()
    ref = oracle.merge_local(a.reshape(2, rows), Ad.reshape(2, rows, 128), Q.reshape(2, rows, 128), qs, qp,
                             Kl.reshape(2, B, T, 128), Vl.reshape(2, B, T, 128), ll, 1 / math.sqrt(128))
    vmax = max(Vl.float().abs().max().item(), Ad.abs().max().item())
    assert np.abs(out.cpu().numpy().reshape(2, rows, 128) - ref).max() <= ATT_TOL * vmax


def test_merge_tc_bad_metadata_flags():
    nx.device_error_flags(clear=True)
    G, nq, B, T = 4, 64, 2, 16
    g = torch.Generator().manual_seed(2)
    Q = torch.randn(1, 1, G, nq, 128, generator=g).to(torch.bfloat16).cuda()
    Kl = torch.randn(1, 1, B, T, 128, generator=g).to(torch.bfloat16).cuda()
    a = torch.zeros(1, 1, G, nq).cuda()
    Ad = torch.randn(1, 1, G, nq, 128).cuda()
    qs = torch.zeros(nq, dtype=torch.int32)
    qs[5] = 7                                                  # not a sequence
    qp = torch.full((nq,), T - 1, dtype=torch.int32)
    ll = torch.tensor([T, T], dtype=torch.int32)
    out = nx.merge_local(a, Ad, Q, qs.cuda(), qp.cuda(), Kl, Kl, ll.cuda())
    assert nx.device_error_flags(clear=True) & 2
    assert torch.equal(out[..., 5, :], Ad[..., 5, :])


def test_split_identity_on_gpu():
    """merge(exact alpha, A) == full attention over document + local (Eq. (3.4))."""
    wl = make_workload("toy", L=1, Hkv=2, G=2, n=1500, nq=6, B=2, T=20, mode="decode", with_modules=False, seed=8)
    wl.q_pos = torch.tensor([19, 4, 0, 13, 19, 7], dtype=torch.int32)
    wl.q_seq = torch.tensor([0, 1, 0, 1, 1, 0], dtype=torch.int32)
    wl.local_len = torch.tensor([20, 14], dtype=torch.int32)
    alpha, A = nx.cache_attn_lse(cuda(wl.K), cuda(wl.V), cuda(wl.Q))
    out = nx.merge_local(alpha, A, cuda(wl.Q), cuda(wl.q_seq), cuda(wl.q_pos), cuda(wl.Kloc), cuda(wl.Vloc),
                         cuda(wl.local_len))
    ref = oracle.full_attention(wl.K.reshape(2, 1500, 128), wl.V.reshape(2, 1500, 128), wl.Q.reshape(2, 12, 128),
                                wl.q_seq, wl.q_pos, wl.Kloc.reshape(2, 2, 20, 128), wl.Vloc.reshape(2, 2, 20, 128),
                                wl.local_len, wl.scale)
    vmax = max(wl.V.float().abs().max().item(), wl.Vloc.float().abs().max().item())
    assert np.abs(out.cpu().numpy().reshape(2, 12, 128) - ref).max() <= ATT_TOL * vmax


# ---------------------------------------------------------------------------
# (ii) module forward
# ---------------------------------------------------------------------------
def module_case(wl):
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    a, At = nx.module_forward(mods, cuda(wl.Q))
    torch.cuda.synchronize()
    ao, Ao = oracle.module_forward(wl)
    a = a.cpu().numpy().reshape(wl.L, wl.Hkv, wl.rows)
    At = At.cpu().numpy().reshape(wl.L, wl.Hkv, wl.rows, 128)
    worst = 0.0
    for (l, h), ref in ao.items():
        ea = np.abs(a[l, h] - ref).max() / max(np.abs(ref).max(), 1e-30)
        eA = np.abs(At[l, h] - Ao[(l, h)]).max() / max(np.abs(Ao[(l, h)]).max(), 1e-30)
        worst = max(worst, ea, eA)
        assert ea <= MLP_TOL and eA <= MLP_TOL, ((l, h), ea, eA)
    return mods, ao, Ao, worst


def test_module_forward_toy():
    wl = make_workload("toy", seed=0)
    module_case(wl)


@pytest.mark.parametrize("kw", [
    dict(L=2, Hkv=2, G=7, nq=10, widths=[208, 96], depth=2),    # ragged H, partial token block
    dict(L=1, Hkv=3, G=2, nq=1, widths=[512], depth=2),         # decode: N = 16 rows
    dict(L=3, Hkv=1, G=4, nq=20, widths=[16, 1024, 144], depth=2),
    dict(L=1, Hkv=2, G=1, nq=33, widths=[64], depth=1),
    dict(L=1, Hkv=1, G=3, nq=7, widths=[128], depth=3),
    # >= 64 rows per KV head: the layer-by-layer grouped-GEMM path
    dict(L=2, Hkv=2, G=7, nq=40, widths=[208, 96], depth=2),    # 280 rows: two ragged row tiles
    dict(L=3, Hkv=1, G=4, nq=300, widths=[16, 1024, 144], depth=3),   # 1200 rows, 5 row tiles
    dict(L=1, Hkv=2, G=1, nq=130, widths=[64], depth=1),        # depth 1: readout straight from h_0
    dict(L=1, Hkv=1, G=2, nq=64, widths=[512], depth=2),        # 128 rows
    dict(L=1, Hkv=2, G=4, nq=16, widths=[256], depth=2),        # exactly 64 rows: the first grouped-GEMM size
    dict(L=1, Hkv=1, G=7, nq=9, widths=[144], depth=2),         # 63 rows: still one CTA per block of tokens
    dict(L=2, Hkv=2, G=2, nq=5, widths=[768, 1024], depth=2),   # >= 1 MB per net: one CTA per net
    dict(L=1, Hkv=1, G=3, nq=4, widths=[1024], depth=3),
    # widths past 8 row tiles (up to NECTAR_MAX_WIDTH = 2048)
    dict(L=2, Hkv=1, G=2, nq=3, widths=[2048, 1152], depth=2),  # one launch, 16 and 9 row tiles
    dict(L=1, Hkv=2, G=7, nq=2, widths=[1152], depth=3),
    dict(L=1, Hkv=1, G=40, nq=1, widths=[2048], depth=2),       # 16 tiles x 48 rows > 512 TMEM columns: GEMM path
    dict(L=1, Hkv=2, G=4, nq=40, widths=[2048], depth=2),       # grouped GEMM, 16 units tiles
    # the API's limits: depth 4 (NECTAR_MAX_DEPTH) on both paths, 256 layers (NECTAR_MAX_LAYERS)
    dict(L=1, Hkv=2, G=2, nq=3, widths=[256], depth=4),         # one launch
    dict(L=1, Hkv=1, G=4, nq=20, widths=[128], depth=4),        # 80 rows: grouped GEMM
    # 256 layers, 16 rows per head (with 2 rows the score readout of a head
    # can cancel towards 0, where the relative measure is ill-posed)
    dict(L=256, Hkv=1, G=2, nq=8, widths=[16, 32, 48, 64] * 64, depth=1),
])
def test_module_forward_shapes(kw):
    kw = dict(kw)
    wl = make_workload("toy", n=16, T=1, with_local=False, with_modules=True, seed=len(kw["widths"]) + kw["G"], **kw)
    module_case(wl)


# ---------------------------------------------------------------------------
# fused decode
# ---------------------------------------------------------------------------
def decode_case(wl):
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = (cuda(wl.Q), cuda(wl.q_seq), cuda(wl.q_pos), cuda(wl.Kloc), cuda(wl.Vloc), cuda(wl.local_len))
    out = nx.decode(mods, *args)
    a, At = nx.module_forward(mods, args[0])
    out2 = nx.merge_local(a, At, *args)
    torch.cuda.synchronize()
    H = wl.heads
    ao, Ao = oracle.module_forward(wl)
    keys = [(l, h) for l in range(wl.L) for h in range(wl.Hkv)]
    a_o = np.stack([ao[k] for k in keys])
    A_o = np.stack([Ao[k] for k in keys])
    ref = oracle.merge_local(a_o, A_o, wl.Q.reshape(H, wl.rows, 128), wl.q_seq, wl.q_pos,
                             wl.Kloc.reshape(H, wl.B, wl.T, 128), wl.Vloc.reshape(H, wl.B, wl.T, 128),
                             wl.local_len, wl.scale)
    got = out.cpu().numpy().reshape(H, wl.rows, 128)
    # bound: |d out| <= |d a| * max|A_theta - out| + |d A_theta| + attention rounding
    da = MLP_TOL * np.abs(a_o).max()
    dA = MLP_TOL * np.abs(A_o).max()
    vmax = max(wl.Vloc.float().abs().max().item(), np.abs(A_o).max())
    bound = da * (np.abs(A_o).max() + np.abs(ref).max()) + dA + ATT_TOL * vmax
    err = np.abs(got - ref).max()
    assert err <= bound, (err, bound)
    # the merge step alone, at the attention tolerance: the GPU's own
    # (a_theta, A_theta) through the oracle's merge (Eqs. (3.4)-(3.5))
    ag = a.cpu().numpy().reshape(H, wl.rows)
    Atg = At.cpu().numpy().reshape(H, wl.rows, 128)
    ref_m = oracle.merge_local(ag, Atg, wl.Q.reshape(H, wl.rows, 128), wl.q_seq, wl.q_pos,
                               wl.Kloc.reshape(H, wl.B, wl.T, 128), wl.Vloc.reshape(H, wl.B, wl.T, 128),
                               wl.local_len, wl.scale)
    vmax_m = max(wl.Vloc.float().abs().max().item(), np.abs(Atg).max())
    err_m = np.abs(got - ref_m).max()
    assert err_m <= ATT_TOL * vmax_m, (err_m, ATT_TOL * vmax_m)
    # fused == unfused on the GPU (same arithmetic, different summation order)
    assert torch.allclose(out, out2, rtol=0, atol=1e-4 * max(1.0, out2.abs().max().item()))


def test_decode_toy_prefill():
    decode_case(make_workload("toy", seed=1))


@pytest.mark.parametrize("kw", [
    dict(L=2, Hkv=2, G=2, n=16, B=3, T=40, widths=[512, 512]),
    dict(L=1, Hkv=2, G=7, n=16, B=10, T=33, widths=[208]),
    dict(L=2, Hkv=1, G=4, n=16, B=20, T=17, widths=[1024, 64]),
    dict(L=1, Hkv=2, G=8, n=16, B=5, T=70, widths=[256]),      # 8 heads per local job
    dict(L=1, Hkv=1, G=12, n=16, B=4, T=45, widths=[128]),     # two local jobs per token (8 + 4 heads)
    dict(L=2, Hkv=2, G=4, n=16, B=40, T=50, widths=[256, 512]),   # 160 rows per KV head: GEMM path
    dict(L=1, Hkv=2, G=7, n=16, B=64, T=33, widths=[768]),     # 448 rows: two row tiles of 224
    dict(L=2, Hkv=2, G=4, n=16, B=16, T=40, widths=[256, 128]),   # exactly 64 rows: grouped-GEMM decode
    dict(L=1, Hkv=2, G=16, n=16, B=8, T=300, widths=[256]),    # 128 rows, 16 heads per local job, 3 tiles
    dict(L=2, Hkv=2, G=2, n=16, B=3, T=40, widths=[768, 896]),   # one CTA per net in the one-launch decode
    dict(L=1, Hkv=2, G=2, n=16, B=3, T=40, widths=[2048]),        # the widest layer, one-launch decode
    dict(L=1, Hkv=1, G=7, n=16, B=16, T=40, widths=[1152]),       # 112 rows: grouped GEMM at 1152 units
    dict(L=1, Hkv=2, G=2, n=16, B=3, T=40, widths=[256], depth=4),   # depth 4: three h exchanges
    dict(L=1, Hkv=1, G=4, n=16, B=20, T=40, widths=[128], depth=4),  # depth 4, 80 rows: grouped GEMM
    dict(L=256, Hkv=1, G=2, n=16, B=1, T=8, widths=[16, 64] * 128, depth=1),   # 256 layers
])
@pytest.mark.parametrize("cluster", ["auto", "0"])
def test_decode_shapes(kw, cluster, monkeypatch):
    # "auto": calls of <= 32 (l, h) pairs and <= 64 rows per head take the
    # cluster decode; "0": the one-launch decode for every shape
    if cluster == "0":
        monkeypatch.setenv("NECTAR_DECODE_CLUSTER", "0")
    wl = make_workload("qwen3_1p7b", seed=2, key_scale=None, **kw)
    wl.local_len = torch.randint(0, wl.T + 1, (wl.B,), generator=torch.Generator().manual_seed(3)).to(torch.int32)
    wl.q_pos = (wl.local_len[wl.q_seq.long()] - 1).clamp(min=0).to(torch.int32)
    decode_case(wl)


# The cluster decode (one cluster per (l, h), hidden units sliced over the
# CTAs holding each net, merge in-cluster) on the shapes it takes: at most 64
# rows per KV head, in its three plans (8 CTAs with one net each: 4 slices
# per net; 8 CTAs with both nets: 8 slices; 16 CTAs with one net each).
# Widths cover 64- and 128-unit slices (512), partial and empty slices (208),
# 128- and 256-unit slices (1024) next to a layer held by one CTA (64), a
# 512-unit slice (2048: four M tiles per CTA), slices that start inside a
# 128-row weight tile (768 and 1152), depths 1 and 3 (no exchange;
# two h buffers), G = 12 (three head blocks of the local warps), 64 rows
# (N = 64).
@pytest.mark.parametrize("kw", [
    dict(L=2, Hkv=2, G=2, n=16, B=3, T=40, widths=[512, 512]),
    dict(L=1, Hkv=2, G=7, n=16, B=2, T=33, widths=[208]),
    dict(L=2, Hkv=1, G=4, n=16, B=5, T=17, widths=[1024, 64]),
    dict(L=2, Hkv=2, G=2, n=16, B=3, T=70, widths=[256, 128], depth=1),
    dict(L=2, Hkv=2, G=2, n=16, B=3, T=70, widths=[256, 384], depth=3),
    dict(L=1, Hkv=1, G=12, n=16, B=4, T=45, widths=[128]),
    dict(L=1, Hkv=2, G=16, n=16, B=4, T=300, widths=[256]),
    dict(L=2, Hkv=2, G=2, n=16, B=1, T=512, widths=[512, 512]),     # the headline's shape per layer
    dict(L=1, Hkv=1, G=4, n=16, B=2, T=64, widths=[2048]),
    dict(L=2, Hkv=1, G=2, n=16, B=2, T=40, widths=[768, 1152]),   # slices that start inside a 128-row tile
])
@pytest.mark.parametrize("cluster", ["8:1", "8:2", "16:1"])
def test_decode_cluster_shapes(kw, cluster, monkeypatch):
    size, nets = cluster.split(":")
    monkeypatch.setenv("NECTAR_DECODE_CLUSTER", size)
    monkeypatch.setenv("NECTAR_DECODE_CLUSTER_NETS", nets)
    wl = make_workload("qwen3_1p7b", seed=7, key_scale=None, **kw)
    wl.local_len = torch.randint(0, wl.T + 1, (wl.B,), generator=torch.Generator().manual_seed(5)).to(torch.int32)
    wl.q_pos = (wl.local_len[wl.q_seq.long()] - 1).clamp(min=0).to(torch.int32)
    decode_case(wl)


def test_decode_cluster_matches_one_launch(monkeypatch):
    # the same decode through the cluster kernel and the one-CTA-per-head
    # kernel: same arithmetic up to the order of the sums
    wl = make_workload("qwen3_1p7b", seed=8, key_scale=None, L=3, Hkv=2, G=2, n=16, B=2, T=100, widths=[512] * 3)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = (cuda(wl.Q), cuda(wl.q_seq), cuda(wl.q_pos), cuda(wl.Kloc), cuda(wl.Vloc), cuda(wl.local_len))
    monkeypatch.setenv("NECTAR_DECODE_CLUSTER", "0")
    o0 = nx.decode(mods, *args)
    for cluster in ("8:1", "8:2", "16:1"):
        size, nets = cluster.split(":")
        monkeypatch.setenv("NECTAR_DECODE_CLUSTER", size)
        monkeypatch.setenv("NECTAR_DECODE_CLUSTER_NETS", nets)
        o1 = nx.decode(mods, *args)
        l1 = nx.decode_layer_out(mods, *args)
        torch.cuda.synchronize()
        assert nx.device_error_flags(clear=True) == 0
        assert torch.allclose(o1, o0, rtol=0, atol=1e-4 * max(1.0, o0.abs().max().item())), cluster
        assert torch.equal(l1, o1.permute(0, 3, 1, 2, 4).reshape(wl.L, wl.nq, wl.Hkv * wl.G, 128).to(torch.bfloat16))


def test_decode_workspace_checked():
    wl = make_workload("toy", seed=4)
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    args = (cuda(wl.Q), cuda(wl.q_seq), cuda(wl.q_pos), cuda(wl.Kloc), cuda(wl.Vloc), cuda(wl.local_len))
    need = nx.decode_workspace_size(mods, wl.G, wl.nq)
    loc = (wl.heads * wl.rows * 130 * 4 + 255) // 256 * 256
    if wl.rows < 64:
        assert need == (wl.heads * wl.rows * 4 + 255) // 256 * 256 + loc
    else:
        assert need == loc + nx.module_workspace_size(mods, wl.G, wl.nq) > loc
    out = torch.full(wl.Q.shape, float("nan"), device="cuda")
    small = torch.empty(need - 4, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="workspace"):
        nx.decode(mods, *args, out=out, workspace=small)
    torch.cuda.synchronize()
    assert torch.isnan(out).all()       # nothing was enqueued
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    nx.decode(mods, *args, out=out, workspace=ws)
    ref = nx.decode(mods, *args)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_binding_refuses_mismatched_buffers():
    """Caller-given outputs and module sets are checked against Q before any
    launch; matching ones are written in place."""
    wl = make_workload("toy", n=100, T=1, with_local=False, with_modules=True, seed=1, L=2, Hkv=2, G=2, nq=5,
                       widths=[64, 64], depth=2)
    K, V, Q = cuda(wl.K), cuda(wl.V), cuda(wl.Q)
    with pytest.raises(ValueError, match="alpha must have shape"):
        nx.cache_attn_lse(K, V, Q, alpha=torch.empty(2, 2, 2, 4, device="cuda"))
    with pytest.raises(ValueError, match="A must be a CUDA tensor"):
        nx.cache_attn_lse(K, V, Q, A=torch.empty(Q.shape))
    with pytest.raises(TypeError, match="workspace must be torch.uint8"):
        nx.cache_attn_lse(K, V, Q, workspace=torch.empty(1024, device="cuda"))
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G)
    with pytest.raises(ValueError, match="module set is for L=1"):
        nx.module_forward(mods.layer(0), Q)
    alpha = torch.empty(Q.shape[:4], device="cuda")
    A = torch.empty(Q.shape, device="cuda")
    got = nx.cache_attn_lse(K, V, Q, alpha=alpha, A=A)
    assert got[0] is alpha and got[1] is A
    ref = nx.cache_attn_lse(K, V, Q)
    torch.cuda.synchronize()
    assert torch.equal(alpha, ref[0]) and torch.equal(A, ref[1])
