"""C-ABI checks that need no GPU: the library loads, exports every function
that include/nectar.h declares, validates arguments on the host, and packs
module weights in the documented layout."""
import ctypes
import math

import numpy as np
import pytest
import torch

import long_context_attention_split_b200 as nx
from nectar_inputs import make_modules


@pytest.fixture(scope="module", autouse=True)
def built():
    from long_context_attention_split_b200 import build
    build.build()


def test_exports_every_header_function():
    names = nx.header_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(nx.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    for n in ["nectar_cache_attn_lse", "nectar_module_forward", "nectar_merge_local", "nectar_decode"]:
        assert n in names


def test_status_strings_and_version():
    L = nx.lib()
    for s in range(5):
        assert L.nectar_status_string(s)
    assert nx.version().count(".") == 2


def test_static_scratch_size_is_the_headers():
    # the size the library reports is the one include/nectar.h states
    import re
    with open(nx.HEADER_PATH) as f:
        m = re.search(r"#define NECTAR_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", f.read())
    assert m, "NECTAR_STATIC_SCRATCH_BYTES not found in the header"
    assert nx.static_scratch_bytes() == int(m.group(1)) << int(m.group(2))


def test_host_validation_without_device():
    L = nx.lib()
    bad_d = nx.Dims(1, 1, 1, 64)
    st = L.nectar_cache_attn_lse(bad_d, None, None, 10, None, 1, 1.0, None, None, None, 0, None)
    assert st == 2 and b"d = 64" in L.nectar_last_error()
    st = L.nectar_cache_attn_lse(nx.Dims(0, 1, 1, 128), None, None, 10, None, 1, 1.0, None, None, None, 0, None)
    assert st == 1
    st = L.nectar_cache_attn_lse(nx.Dims(1, 1, 1, 128), None, None, -1, None, 1, 1.0, None, None, None, 0, None)
    assert st == 1
    # nq == 0 is a no-op even with no buffers
    assert L.nectar_cache_attn_lse(nx.Dims(1, 1, 1, 128), None, None, 5, None, 0, 1.0, None, None, None, 0, None) == 0
    assert L.nectar_cache_attn_workspace_size(bad_d, 10, 1) == 0
    st = L.nectar_merge_local(nx.Dims(1, 1, 1, 128), None, None, None, 1, None, None, None, None, 1, 1, None, 1.0,
                              None, None)
    assert st == 1
    w = (ctypes.c_int32 * 2)(64, 40)      # 40 is not a multiple of 16
    assert L.nectar_module_packed_elems(nx.Dims(2, 1, 1, 128), 2, w) == 0
    w = (ctypes.c_int32 * 1)(2064)        # too wide
    assert L.nectar_module_packed_elems(nx.Dims(1, 1, 1, 128), 2, w) == 0
    w = (ctypes.c_int32 * 1)(64)
    assert L.nectar_module_packed_elems(nx.Dims(1, 1, 1, 128), 0, w) == 0
    # the bounded-wait self-check takes 1 us .. 1 s, checked before any launch
    for bad in (0, -1, 1000001):
        assert L.nectar_check_wait_timeout(bad, None) == 1
        assert b"limit_us" in L.nectar_last_error()


# -- independent reader of the packed layout (as documented in module_layout.h) --
def r64(x):
    return (x + 63) // 64 * 64


def kch(K):
    return (K + 63) // 64


def read_chunked(blob, off, rows, K):
    """Tiled [ceil(rows/128)][ceil(K/64)][tile rows][64], the 16-byte pieces of
    row i stored in 128-byte-swizzle order (piece j at slot j ^ (i % 8))
    -> dense [rows][K]."""
    out = []
    for m in range((rows + 127) // 128):
        tr = min(128, rows - 128 * m)
        n = kch(K) * tr * 64
        a = blob[off:off + n].reshape(kch(K), tr, 8, 8)
        slot = np.arange(8)[None, :] ^ (np.arange(tr)[:, None] % 8)      # [row][piece] -> stored slot
        a = np.take_along_axis(a, np.broadcast_to(slot[None, :, :, None], a.shape), axis=2)
        out.append(np.concatenate(list(a.reshape(kch(K), tr, 64)), axis=1)[:, :K])
        off += n
    return np.concatenate(out, axis=0), off


def read_net(blob, off, H, depth, dout, d=128):
    out = {"W": [], "b": []}
    for k in range(depth):
        Kk = d if k == 0 else d + H
        W, off = read_chunked(blob, off, H, Kk)
        out["W"].append(W)
        out["b"].append(blob[off:off + H]); off += r64(H)
    if dout == 1:
        out["Wout"] = blob[off:off + H][None]; off += r64(H)
        out["c"] = blob[off:off + 1]; off += 64
    else:
        W, off = read_chunked(blob, off, d, H)
        out["Wout"] = W
        out["c"] = blob[off:off + d]; off += d
    return out, off


@pytest.mark.parametrize("widths,depth,hkv", [([64, 32], 2, 2), ([48], 3, 1), ([16, 208], 1, 3), ([272], 2, 1),
                                               ([96, 2048], 4, 1)])   # the depth and width limits
def test_pack_layout(widths, depth, hkv):
    mods = make_modules(len(widths), hkv, widths, 128, seed=3, device="cpu", depth=depth)
    ms = nx.pack_modules(mods, widths, depth, hkv, G=2, device=None)
    blob = ms.blob.float().numpy()
    assert ms.blob.numel() == nx.packed_elems(len(widths), hkv, 2, widths, depth)
    off = 0
    for l, H in enumerate(widths):
        for h in range(hkv):
            for name, dout in (("score", 1), ("target", 128)):
                net = mods[l][name]
                got, off = read_net(blob, off, H, depth, dout)
                for k in range(depth):
                    if k == 0:
                        ref = net["U"][0][h].float().numpy()
                    else:
                        ref = np.concatenate([net["V"][k][h].float().numpy(), net["U"][k][h].float().numpy()], 1)
                    np.testing.assert_array_equal(got["W"][k], ref)
                    np.testing.assert_array_equal(got["b"][k], net["b"][k][h].float().numpy())
                np.testing.assert_array_equal(got["Wout"], net["Wout"][h].float().numpy())
                np.testing.assert_array_equal(got["c"], net["c"][h].float().numpy())
    assert off == blob.size
    # padding (K columns beyond d + H inside the last chunk) is zero
    H = widths[0]
    if depth >= 2 and (128 + H) % 64:
        W1, _ = read_chunked(blob, r64(0) + kch(128) * H * 64 + r64(H), H, r64(128 + H))
        assert np.all(W1[:, 128 + H:] == 0)


def test_arch_packing_without_backbone_is_the_classic_blob():
    # host-only: nectar_module_pack_arch with D_b = 0 and equal nets writes the
    # classic nectar_module_pack blob, element for element
    from nectar_inputs import make_modules, make_modules_general
    import long_context_attention_split_b200 as nx
    widths = [48, 32, 1024]
    classic = nx.pack_modules(make_modules(3, 2, widths, 128, 5, "cpu", depth=3), widths, 3, 2, 2, device=None)
    mods = make_modules_general(3, 2, 128, 5, "cpu", (0, 3, 3), [], widths, widths)
    arch = nx.pack_modules_arch(mods, nx.Arch((0, 3, 3), [], widths, widths), 2, 2, device=None)
    assert torch.equal(classic.blob, arch.blob)
    # a backbone makes the blob bigger by exactly its layers
    wb = [64, 16, 32]
    with_bb = nx.Arch((1, 3, 3), wb, widths, widths)
    assert with_bb.packed_elems(2) > nx.Arch((0, 3, 3), [], widths, widths).packed_elems(2)


def test_arch_validation_on_the_host():
    # depths and widths outside the supported set are refused (0 elements)
    import long_context_attention_split_b200 as nx
    ok = nx.Arch((2, 1, 2), [64, 32], [32, 16], [48, 96])
    assert ok.packed_elems(2) > 0
    for depths, wb, ws, wt in [((2, 0, 2), [64, 32], [32, 16], [48, 96]),     # a branch without layers
                               ((0, 1, 0), [], [32, 16], [48, 96]),
                               ((3, 1, 2), [64, 32], [32, 16], [48, 96]),     # chain of 5 > NECTAR_MAX_DEPTH
                               ((1, 1, 1), [64, 40], [32, 16], [48, 96]),     # width not a multiple of 16
                               ((0, 2, 2), [], [32, 2064], [48, 96]),         # width above the maximum
                               ((-1, 1, 1), [], [32, 16], [48, 96])]:
        assert nx.Arch(depths, wb, ws, wt).packed_elems(2) == 0, depths


def a256(x):
    return (x + 255) // 256 * 256


def _host_set(L, Hkv, widths, depth, arch=None):
    # the size functions read only the shapes: a host blob of the packed size will do
    if arch is not None:
        n = arch.packed_elems(Hkv)
        return nx.ModuleSet(torch.zeros(n, dtype=torch.bfloat16), arch.width_s, arch.depths[1], L, Hkv, arch=arch)
    n = nx.packed_elems(L, Hkv, 1, widths, depth)
    return nx.ModuleSet(torch.zeros(n, dtype=torch.bfloat16), widths, depth, L, Hkv)


@pytest.mark.parametrize("widths,depth", [([256, 512, 384], 2), ([208, 144, 80], 1), ([128, 128, 1024], 3),
                                          ([2048, 1152], 2)])
@pytest.mark.parametrize("G,nq", [(2, 1), (4, 8), (2, 32), (8, 40), (40, 1)])
def test_workspace_sizes_follow_the_header(widths, depth, G, nq):
    """nectar_module_workspace_size, nectar_decode_workspace_size and
    nectar_decode_layer_out_workspace_size equal the formulas include/nectar.h
    states for them (classic sets; 64 query rows per KV head or more, or
    widths whose 128-unit tiles for round16(G) rows exceed 512 TMEM columns,
    take the layer-by-layer path)."""
    L, Hkv, d = len(widths), 2, 128
    mods = _host_set(L, Hkv, widths, depth)
    rows = L * Hkv * G * nq
    gemm = G * nq >= 64 or math.ceil(max(widths) / 128) * (-(-G // 16) * 16) > 512
    Hp = r64(max(widths))
    mod_ws = ((2 if depth >= 2 else 1) * a256(2 * rows * Hp * 2) + a256(rows * math.ceil(max(widths) / 128) * 4)
              if gemm else 0)
    assert nx.module_workspace_size(mods, G, nq) == mod_ws
    loc = a256(rows * (d + 2) * 4)
    dec_ws = loc + (mod_ws if gemm else a256(rows * 4))
    assert nx.decode_workspace_size(mods, G, nq) == dec_ws
    lo = int(nx.lib().nectar_decode_layer_out_workspace_size(nx.Dims(L, Hkv, G, d), mods.c(), nq))
    assert lo == dec_ws + (0 if gemm else a256(rows * d * 4))


@pytest.mark.parametrize("depths", [(2, 1, 2), (0, 2, 3), (1, 1, 1)])
def test_workspace_sizes_of_backbone_sets(depths):
    """A set with a backbone or unequal nets takes the layer-by-layer path at
    any row count; its chain has D_b + max(D_s, D_t) hidden layers and Hp is
    the widest layer of any part."""
    L, Hkv, G, nq, d = 2, 2, 2, 1, 128
    wb = [640, 256] if depths[0] else []
    arch = nx.Arch(depths, wb, [384, 192], [512, 1008])
    mods = _host_set(L, Hkv, None, None, arch)
    rows = L * Hkv * G * nq
    S = depths[0] + max(depths[1], depths[2])
    Hp = r64(max([384, 192, 512, 1008] + wb))
    mod_ws = (2 if S >= 2 else 1) * a256(2 * rows * Hp * 2) + a256(rows * math.ceil(384 / 128) * 4)
    assert nx.module_workspace_size(mods, G, nq) == mod_ws
    assert nx.decode_workspace_size(mods, G, nq) == a256(rows * (d + 2) * 4) + mod_ws


def test_cache_attn_workspace_needs_a_device():
    """The exact-attention scratch is planned for the current device's SM
    count: with no device the size is 0 (and the compute call fails)."""
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert nx.cache_attn_workspace_size(2, 2, 2, 4096, 1) == 0
    dims = nx.Dims(2, 2, 2, 128)
    assert nx.lib().nectar_quadrature_workspace_size(dims, 512, 1) == 0


def _toy_host_inputs(L=2, Hkv=2, G=2, nq=3, n=16, B=2, T=8):
    bf = torch.bfloat16
    K = torch.zeros(L, Hkv, n, 128, dtype=bf)
    Q = torch.zeros(L, Hkv, G, nq, 128, dtype=bf)
    loc = (torch.zeros(nq, dtype=torch.int32), torch.zeros(nq, dtype=torch.int32),
           torch.zeros(L, Hkv, B, T, 128, dtype=bf), torch.zeros(L, Hkv, B, T, 128, dtype=bf),
           torch.full((B,), T, dtype=torch.int32))
    a = torch.zeros(L, Hkv, G, nq)
    A = torch.zeros(L, Hkv, G, nq, 128)
    return K, Q, loc, a, A


def test_binding_refuses_host_tensors():
    """No compute call runs on host memory: the library sees raw pointers,
    so the binding refuses CPU tensors instead of passing them on (and there
    is no CPU fallback to take instead)."""
    K, Q, loc, a, A = _toy_host_inputs()
    mods = _host_set(2, 2, [64, 64], 2)
    calls = [
        lambda: nx.cache_attn_lse(K, K, Q),
        lambda: nx.cache_attn_lse_static(K, K, Q),
        lambda: nx.module_forward(mods, Q),
        lambda: nx.merge_local(a, A, Q, *loc),
        lambda: nx.decode(mods, Q, *loc),
        lambda: nx.decode_layer_out(mods, Q, *loc),
        lambda: nx.quadrature_init(K, K, 4),
        lambda: nx.quadrature_forward(K, K, Q),
        lambda: nx.fit_metrics(a, A, a, A, Q),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()


class _SeenAsCuda(torch.Tensor):
    """A host tensor that claims to be on a CUDA device, so that the checks
    after the device check can be reached on a machine without one.  Every
    case below is refused before the library is called."""

    @property
    def is_cuda(self):
        return True


def test_binding_checks_shapes_and_dtypes():
    """Inputs and caller-given outputs must have the shapes the call implies:
    a short buffer would otherwise be read or written past its end."""
    K, Q, loc, a, A = (x.as_subclass(_SeenAsCuda) if isinstance(x, torch.Tensor)
                       else tuple(t.as_subclass(_SeenAsCuda) for t in x) for x in _toy_host_inputs())
    with pytest.raises(ValueError, match="K must have shape"):
        nx.cache_attn_lse(K[:1], K[:1], Q)                       # one layer of cache, two of queries
    with pytest.raises(ValueError, match="V must have shape"):
        nx.cache_attn_lse(K, K[:, :, :8], Q)                     # V shorter than K
    with pytest.raises(ValueError, match="Kloc must have shape"):
        nx.merge_local(a, A, Q, loc[0], loc[1], loc[2][:, :1], loc[3], loc[4])
    with pytest.raises(ValueError, match="local_len must have shape"):
        nx.merge_local(a, A, Q, loc[0], loc[1], loc[2], loc[3], loc[4][:1])
    with pytest.raises(ValueError, match="q_pos must have shape"):
        nx.merge_local(a, A, Q, loc[0], loc[1][:2], loc[2], loc[3], loc[4])
    with pytest.raises(ValueError, match="a must have shape"):
        nx.fit_metrics(a, A, a[:, :, :1], A, Q)
    with pytest.raises(TypeError, match="A_theta must be torch.float32"):
        nx.fit_metrics(a, A, a, A.double(), Q)
    with pytest.raises(ValueError, match="Q must be a tensor"):
        nx.module_forward(_host_set(2, 2, [64, 64], 2), Q[0])
    with pytest.raises(ValueError, match="out must have shape"):
        nx._out(torch.zeros(3), "out", torch.float32, (2, 2), None)
    with pytest.raises(ValueError, match="module set is for L=1"):
        nx._need_mods(_host_set(1, 2, [64], 2), nx.Dims(2, 2, 2, 128))
    with pytest.raises(ValueError, match="module weights must be on a CUDA device"):
        nx._need_mods(_host_set(2, 2, [64, 64], 2), nx.Dims(2, 2, 2, 128))


def test_plain_c_client(tmp_path):
    """The boundary is usable from C alone: tests/c_client/c_client.c
    includes only include/nectar.h (C99, -pedantic -Werror), links
    libnectar.so and exercises the entry points that need no GPU, and the
    per-thread error text from two threads at once."""
    import os
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(nx.LIB_PATH)
    exe = str(tmp_path / "c_client")
    r = subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                        "-I", os.path.join(root, "include"), os.path.join(root, "tests", "c_client", "c_client.c"),
                        "-L", libdir, "-lnectar", f"-Wl,-rpath,{libdir}", "-pthread", "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok "), r.stdout + r.stderr


def test_layer_depth_and_width_limits_on_the_host():
    """NECTAR_MAX_LAYERS, NECTAR_MAX_DEPTH and NECTAR_MAX_WIDTH: the limit
    itself is accepted, one past it is refused with the reason."""
    L = nx.lib()
    assert nx.packed_elems(256, 1, 1, [16] * 256, 1) > 0
    assert nx.packed_elems(257, 1, 1, [16] * 257, 1) <= 0
    assert b"L = 257" in L.nectar_last_error()
    assert nx.packed_elems(1, 1, 1, [2048], 4) > 0
    assert nx.packed_elems(1, 1, 1, [64], 5) <= 0
    assert b"depth 5" in L.nectar_last_error()
    assert nx.packed_elems(1, 1, 1, [2064], 2) <= 0
    # a backbone chain counts against the depth limit as a whole
    assert nx.Arch((2, 2, 1), [64], [64], [64]).packed_elems(1) > 0
    assert nx.Arch((2, 3, 1), [64], [64], [64]).packed_elems(1) <= 0
