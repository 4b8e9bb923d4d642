"""Nectar hot path on B200: Python binding of libnectar.so.

Argument marshalling only -- every step of the path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the stream.  The entry
points mirror include/nectar.h:

    cache_attn_lse   (i)   exact alpha(q), A(q) of Eq. (3.1) over the document
    module_forward   (ii)  score / target MLPs a_theta, A_theta of Eq. (3.6)
    merge_local      (iii) merge with exact causal local attention, Eqs. (3.4)-(3.5)
    decode           (ii)+(iii) in one launch

"Nectar: Neural Estimation of Cached-Token Attention via Regression"
(Monteiro, Klein, Ablin, Cuturi).
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from typing import List, Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnectar.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "nectar.h")

NECTAR_MAX_DEPTH = 4
STATUS = {0: "NECTAR_OK", 1: "NECTAR_ERR_INVALID_ARG", 2: "NECTAR_ERR_UNSUPPORTED",
          3: "NECTAR_ERR_WORKSPACE", 4: "NECTAR_ERR_CUDA"}


class NectarError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("G", ctypes.c_int32), ("d", ctypes.c_int32)]


class _ArchC(ctypes.Structure):
    _fields_ = [("depth_b", ctypes.c_int32), ("depth_s", ctypes.c_int32), ("depth_t", ctypes.c_int32),
                ("width_b", ctypes.POINTER(ctypes.c_int32)), ("width_s", ctypes.POINTER(ctypes.c_int32)),
                ("width_t", ctypes.POINTER(ctypes.c_int32))]


class _ModuleSetC(ctypes.Structure):
    _fields_ = [("depth", ctypes.c_int32), ("width", ctypes.POINTER(ctypes.c_int32)),
                ("weights", ctypes.c_void_p), ("weights_elems", ctypes.c_int64),
                ("arch", ctypes.POINTER(_ArchC))]


class _NetHostC(ctypes.Structure):
    _fields_ = [("U", ctypes.c_void_p * NECTAR_MAX_DEPTH), ("V", ctypes.c_void_p * NECTAR_MAX_DEPTH),
                ("b", ctypes.c_void_p * NECTAR_MAX_DEPTH), ("Wout", ctypes.c_void_p), ("c", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnectar.so (built in-tree by build.py).  Raises if it is missing:
    there is no fallback path."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m long_context_attention_split_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    S = ctypes.c_int
    L.nectar_cache_attn_workspace_size.argtypes = [Dims, I64, I64]
    L.nectar_cache_attn_workspace_size.restype = ctypes.c_size_t
    L.nectar_cache_attn_lse.argtypes = [Dims, P, P, I64, P, I64, F, P, P, P, ctypes.c_size_t, P]
    L.nectar_cache_attn_lse.restype = S
    L.nectar_cache_attn_lse_static.argtypes = [Dims, P, P, I64, P, I64, F, P, P, P]
    L.nectar_cache_attn_lse_static.restype = S
    L.nectar_static_scratch_bytes.argtypes = []
    L.nectar_static_scratch_bytes.restype = ctypes.c_size_t
    L.nectar_module_packed_elems.argtypes = [Dims, I32, P]
    L.nectar_module_packed_elems.restype = I64
    L.nectar_module_pack.argtypes = [Dims, I32, P, P, P, I64]
    L.nectar_module_pack.restype = S
    L.nectar_module_packed_elems_arch.argtypes = [Dims, ctypes.POINTER(_ArchC)]
    L.nectar_module_packed_elems_arch.restype = I64
    L.nectar_module_pack_arch.argtypes = [Dims, ctypes.POINTER(_ArchC), P, P, I64]
    L.nectar_module_pack_arch.restype = S
    L.nectar_module_workspace_size.argtypes = [Dims, ctypes.POINTER(_ModuleSetC), I64]
    L.nectar_module_workspace_size.restype = ctypes.c_size_t
    L.nectar_module_forward.argtypes = [Dims, ctypes.POINTER(_ModuleSetC), P, I64, P, P, P, ctypes.c_size_t, P]
    L.nectar_module_forward.restype = S
    L.nectar_merge_local.argtypes = [Dims, P, P, P, I64, P, P, P, P, I32, I32, P, F, P, P]
    L.nectar_merge_local.restype = S
    L.nectar_decode_workspace_size.argtypes = [Dims, ctypes.POINTER(_ModuleSetC), I64]
    L.nectar_decode_workspace_size.restype = ctypes.c_size_t
    L.nectar_decode.argtypes = [Dims, ctypes.POINTER(_ModuleSetC), P, I64, P, P, P, P, I32, I32, P, F, P, P,
                                ctypes.c_size_t, P]
    L.nectar_decode.restype = S
    L.nectar_decode_layer_out_workspace_size.argtypes = [Dims, ctypes.POINTER(_ModuleSetC), I64]
    L.nectar_decode_layer_out_workspace_size.restype = ctypes.c_size_t
    L.nectar_decode_layer_out.argtypes = [Dims, ctypes.POINTER(_ModuleSetC), P, I64, P, P, P, P, I32, I32, P, F, P,
                                          P, ctypes.c_size_t, P]
    L.nectar_decode_layer_out.restype = S
    L.nectar_quadrature_init.argtypes = [Dims, P, P, I64, I64, P, P, P]
    L.nectar_quadrature_init.restype = S
    L.nectar_quadrature_workspace_size.argtypes = [Dims, I64, I64]
    L.nectar_quadrature_workspace_size.restype = ctypes.c_size_t
    L.nectar_quadrature_forward.argtypes = [Dims, P, P, I64, P, I64, F, P, P, P, ctypes.c_size_t, P]
    L.nectar_quadrature_forward.restype = S
    L.nectar_fit_metrics.argtypes = [Dims, I64, P, P, P, P, P, P, P]
    L.nectar_fit_metrics.restype = S
    L.nectar_status_string.argtypes = [S]
    L.nectar_status_string.restype = ctypes.c_char_p
    L.nectar_last_error.restype = ctypes.c_char_p
    L.nectar_device_error_flags.argtypes = [ctypes.POINTER(ctypes.c_int32), I32]
    L.nectar_device_error_flags.restype = S
    L.nectar_version.restype = ctypes.c_char_p
    L.nectar_check_wait_timeout.argtypes = [I32, P]
    L.nectar_check_wait_timeout.restype = S
    _lib = L
    return L


def header_functions() -> List[str]:
    """Names of the functions declared in include/nectar.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nectar_[a-z0-9_]+)\s*\(", text)))


def _check(status: int, what: str) -> None:
    if status != 0:
        raise NectarError(status, f"{what}: {lib().nectar_last_error().decode()}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None, device=None) -> None:
    """Checks that the library can take `t` as a pointer to `shape` elements
    of `dtype` in CUDA memory: the C ABI sees only the pointer, so a host
    tensor or a short buffer must be refused here."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} must have shape {tuple(int(x) for x in shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call runs on {device}")


def _out(t: Optional[torch.Tensor], name: str, dtype, shape, device) -> torch.Tensor:
    """A caller's output tensor, checked, or a new one."""
    if t is None:
        return torch.empty(tuple(shape), dtype=dtype, device=device)
    _need(t, name, dtype, shape, device)
    return t


def _workspace(t: Optional[torch.Tensor], nbytes: int, device) -> Optional[torch.Tensor]:
    """A caller's workspace (uint8, its size is checked by the library), or a
    new one of `nbytes` when needed."""
    if t is None:
        return torch.empty(nbytes, dtype=torch.uint8, device=device) if nbytes > 0 else None
    _need(t, "workspace", torch.uint8, device=device)
    return t


def _need_mods(mods: "ModuleSet", dims: Dims) -> None:
    if not isinstance(mods, ModuleSet):
        raise TypeError(f"mods must be a ModuleSet, got {type(mods).__name__}")
    if (mods.L, mods.Hkv) != (dims.L, dims.Hkv):
        raise ValueError(f"module set is for L={mods.L}, Hkv={mods.Hkv}; Q has L={dims.L}, Hkv={dims.Hkv}")
    if mods.blob.device.type != "cuda":
        raise ValueError("module weights must be on a CUDA device")


def dims_of(Q: torch.Tensor) -> Tuple[Dims, int]:
    """Q: [L][Hkv][G][nq][d] -> (dims, nq)."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 5:
        raise ValueError("Q must be a tensor [L, Hkv, G, nq, d]")
    L_, Hkv, G, nq, d = Q.shape
    return Dims(L_, Hkv, G, d), nq


def version() -> str:
    return lib().nectar_version().decode()


# ---------------------------------------------------------------------------
# (i) exact cached-token attention
# ---------------------------------------------------------------------------
def cache_attn_workspace_size(L: int, Hkv: int, G: int, n: int, nq: int, d: int = 128) -> int:
    return int(lib().nectar_cache_attn_workspace_size(Dims(L, Hkv, G, d), n, nq))


def _cache_args(K, V, Q, dims: Dims) -> int:
    """Checks K, V [L, Hkv, n, d] against Q [L, Hkv, G, nq, d]; returns n."""
    _need(Q, "Q", torch.bfloat16)
    if not isinstance(K, torch.Tensor) or K.dim() != 4:
        raise ValueError("K must be a tensor [L, Hkv, n, d]")
    n = K.shape[2]
    for t, nm in ((K, "K"), (V, "V")):
        _need(t, nm, torch.bfloat16, (dims.L, dims.Hkv, n, dims.d), Q.device)
    return n


def cache_attn_lse(K, V, Q, scale: Optional[float] = None, alpha=None, A=None, workspace=None, stream=None):
    """alpha [L,Hkv,G,nq] fp32 and A [L,Hkv,G,nq,d] fp32 of Eq. (3.1).

    K, V: bf16 [L, Hkv, n, d]; Q: bf16 [L, Hkv, G, nq, d] (CUDA)."""
    dims, nq = dims_of(Q)
    n = _cache_args(K, V, Q, dims)
    if scale is None:
        scale = 1.0 / math.sqrt(dims.d)
    alpha = _out(alpha, "alpha", torch.float32, Q.shape[:4], Q.device)
    A = _out(A, "A", torch.float32, Q.shape, Q.device)
    workspace = _workspace(workspace, cache_attn_workspace_size(dims.L, dims.Hkv, dims.G, n, nq, dims.d), Q.device)
    st = lib().nectar_cache_attn_lse(dims, _ptr(K), _ptr(V), n, _ptr(Q), nq, float(scale), _ptr(alpha), _ptr(A),
                                     _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                     _stream(stream))
    _check(st, "nectar_cache_attn_lse")
    return alpha, A


def cache_attn_lse_static(K, V, Q, scale: Optional[float] = None, alpha=None, A=None, stream=None):
    """As cache_attn_lse, through nectar_cache_attn_lse_static: no workspace is
    passed or allocated; the library's fixed device scratch area is used."""
    dims, nq = dims_of(Q)
    n = _cache_args(K, V, Q, dims)
    if scale is None:
        scale = 1.0 / math.sqrt(dims.d)
    alpha = _out(alpha, "alpha", torch.float32, Q.shape[:4], Q.device)
    A = _out(A, "A", torch.float32, Q.shape, Q.device)
    st = lib().nectar_cache_attn_lse_static(dims, _ptr(K), _ptr(V), n, _ptr(Q), nq, float(scale), _ptr(alpha),
                                            _ptr(A), _stream(stream))
    _check(st, "nectar_cache_attn_lse_static")
    return alpha, A


def static_scratch_bytes() -> int:
    """Size of the library's static scratch area (what
    nectar_cache_attn_lse_static can use), as the library reports it."""
    return int(lib().nectar_static_scratch_bytes())


# ---------------------------------------------------------------------------
# module set
# ---------------------------------------------------------------------------
class Arch:
    """Depths (D_b, D_s, D_t) and per-layer widths of a module set with a
    shared backbone (nectar_module_arch)."""

    def __init__(self, depths: Sequence[int], width_b: Sequence[int], width_s: Sequence[int],
                 width_t: Sequence[int]):
        self.depths = tuple(int(x) for x in depths)
        self.width_b = [int(w) for w in width_b]
        self.width_s = [int(w) for w in width_s]
        self.width_t = [int(w) for w in width_t]
        i32 = ctypes.POINTER(ctypes.c_int32)
        self._wb = (ctypes.c_int32 * max(len(self.width_b), 1))(*self.width_b)
        self._ws = (ctypes.c_int32 * len(self.width_s))(*self.width_s)
        self._wt = (ctypes.c_int32 * len(self.width_t))(*self.width_t)
        self._c = _ArchC(self.depths[0], self.depths[1], self.depths[2], ctypes.cast(self._wb, i32),
                         ctypes.cast(self._ws, i32), ctypes.cast(self._wt, i32))

    def layers(self, lo: int, hi: int) -> "Arch":
        return Arch(self.depths, self.width_b[lo:hi] if self.depths[0] else [], self.width_s[lo:hi],
                    self.width_t[lo:hi])

    def packed_elems(self, Hkv: int, d: int = 128) -> int:
        return int(lib().nectar_module_packed_elems_arch(Dims(len(self.width_s), Hkv, 1, d), ctypes.byref(self._c)))


class ModuleSet:
    """A packed module set on the device (nectar_module_set): the classic
    one (both nets `depth` layers of `widths`) or, with `arch`, one with a
    shared backbone and nets of their own depths and widths."""

    def __init__(self, blob: torch.Tensor, widths: Sequence[int], depth: int, L: int, Hkv: int,
                 arch: Optional[Arch] = None):
        self.blob = blob
        self.widths = [int(w) for w in widths]
        self.depth = int(depth)
        self.L, self.Hkv = L, Hkv
        self.arch = arch
        self._w = (ctypes.c_int32 * max(len(self.widths), 1))(*self.widths)
        self._c = _ModuleSetC(self.depth, ctypes.cast(self._w, ctypes.POINTER(ctypes.c_int32)),
                              blob.data_ptr(), blob.numel(),
                              ctypes.pointer(arch._c) if arch is not None else None)

    def c(self):
        return ctypes.byref(self._c)

    @property
    def bytes(self) -> int:
        return self.blob.numel() * 2

    def layer(self, l: int) -> "ModuleSet":
        """The modules of layer l alone, as a one-layer set viewing the same
        blob (blocks are stored layer after layer)."""
        if self.arch is not None:
            off = self.arch.layers(0, l).packed_elems(self.Hkv) if l > 0 else 0
            one = self.arch.layers(l, l + 1)
            n = one.packed_elems(self.Hkv)
            return ModuleSet(self.blob[off:off + n], self.widths[l:l + 1], self.depth, 1, self.Hkv, arch=one)
        off = packed_elems(l, self.Hkv, 1, self.widths[:l], self.depth) if l > 0 else 0
        n = packed_elems(1, self.Hkv, 1, self.widths[l:l + 1], self.depth)
        return ModuleSet(self.blob[off:off + n], self.widths[l:l + 1], self.depth, 1, self.Hkv)


def packed_elems(L: int, Hkv: int, G: int, widths: Sequence[int], depth: int, d: int = 128) -> int:
    w = (ctypes.c_int32 * L)(*widths)
    return int(lib().nectar_module_packed_elems(Dims(L, Hkv, G, d), depth, w))


def pack_modules(modules, widths: Sequence[int], depth: int, Hkv: int, G: int, d: int = 128,
                 device="cuda") -> ModuleSet:
    """Pack per-layer nets (dicts with U, V, b, Wout, c as bf16 tensors with a
    leading Hkv axis) with nectar_module_pack and copy the blob to `device`."""
    L_ = len(modules)
    total = packed_elems(L_, Hkv, G, widths, depth, d)
    if total <= 0:
        raise NectarError(1, lib().nectar_last_error().decode())
    blob = torch.zeros(total, dtype=torch.bfloat16)
    keep = []
    nets = (_NetHostC * (2 * L_))()
    for l, layer in enumerate(modules):
        for j, name in enumerate(("score", "target")):
            net = layer[name]
            nh = nets[2 * l + j]
            for k in range(depth):
                u = net["U"][k].detach().cpu().contiguous()
                b = net["b"][k].detach().cpu().contiguous()
                keep += [u, b]
                nh.U[k] = u.data_ptr()
                nh.b[k] = b.data_ptr()
                if k > 0:
                    v = net["V"][k].detach().cpu().contiguous()
                    keep.append(v)
                    nh.V[k] = v.data_ptr()
            wo = net["Wout"].detach().cpu().contiguous()
            cc = net["c"].detach().cpu().contiguous()
            keep += [wo, cc]
            nh.Wout, nh.c = wo.data_ptr(), cc.data_ptr()
    w = (ctypes.c_int32 * L_)(*widths)
    st = lib().nectar_module_pack(Dims(L_, Hkv, G, d), depth, w, nets, blob.data_ptr(), total)
    _check(st, "nectar_module_pack")
    dev_blob = blob.to(device) if device is not None else blob
    return ModuleSet(dev_blob, widths, depth, L_, Hkv)


def pack_modules_arch(modules, arch: Arch, Hkv: int, G: int, d: int = 128, device="cuda") -> ModuleSet:
    """Pack per-layer module sets with a shared backbone (dicts "backbone",
    "score", "target" with U, V, b lists, and Wout, c for the branches; V[k]
    None for a layer that starts a chain) with nectar_module_pack_arch and
    copy the blob to `device`."""
    L_ = len(modules)
    dims = Dims(L_, Hkv, G, d)
    total = int(lib().nectar_module_packed_elems_arch(dims, ctypes.byref(arch._c)))
    if total <= 0:
        raise NectarError(1, lib().nectar_last_error().decode())
    blob = torch.zeros(total, dtype=torch.bfloat16)
    keep = []
    nets = (_NetHostC * (3 * L_))()

    def ptr(t):
        t = t.detach().cpu().contiguous()
        keep.append(t)
        return t.data_ptr()

    for l, layer in enumerate(modules):
        for j, name in enumerate(("backbone", "score", "target")):
            part = layer[name]
            nh = nets[3 * l + j]
            for k in range(len(part["U"])):
                nh.U[k] = ptr(part["U"][k])
                nh.b[k] = ptr(part["b"][k])
                if part["V"][k] is not None:
                    nh.V[k] = ptr(part["V"][k])
            if name != "backbone":
                nh.Wout, nh.c = ptr(part["Wout"]), ptr(part["c"])
    st = lib().nectar_module_pack_arch(dims, ctypes.byref(arch._c), nets, blob.data_ptr(), total)
    _check(st, "nectar_module_pack_arch")
    dev_blob = blob.to(device) if device is not None else blob
    return ModuleSet(dev_blob, arch.width_s, arch.depths[1], L_, Hkv, arch=arch)


# ---------------------------------------------------------------------------
# (ii) module forward, (iii) merge, fused decode
# ---------------------------------------------------------------------------
def module_workspace_size(mods: ModuleSet, G: int, nq: int, d: int = 128) -> int:
    return int(lib().nectar_module_workspace_size(Dims(mods.L, mods.Hkv, G, d), mods.c(), nq))


def module_forward(mods: ModuleSet, Q, a=None, A_theta=None, workspace=None, stream=None):
    """(a [L,Hkv,G,nq], A_theta [L,Hkv,G,nq,d]) fp32 for every query row.
    workspace: uint8 CUDA tensor of module_workspace_size(...) bytes (made
    here when None and needed)."""
    dims, nq = dims_of(Q)
    _need(Q, "Q", torch.bfloat16)
    _need_mods(mods, dims)
    a = _out(a, "a", torch.float32, Q.shape[:4], Q.device)
    A_theta = _out(A_theta, "A_theta", torch.float32, Q.shape, Q.device)
    workspace = _workspace(workspace, module_workspace_size(mods, dims.G, nq, dims.d), Q.device)
    st = lib().nectar_module_forward(dims, mods.c(), _ptr(Q), nq, _ptr(a), _ptr(A_theta), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "nectar_module_forward")
    return a, A_theta


def _local_args(q_seq, q_pos, Kloc, Vloc, local_len, Q):
    """Checks the local caches Kloc, Vloc [L, Hkv, B, T, d], q_seq, q_pos [nq]
    and local_len [B] against Q [L, Hkv, G, nq, d]; returns (B, T)."""
    L_, Hkv, _, nq, d = Q.shape
    if not isinstance(Kloc, torch.Tensor) or Kloc.dim() != 5:
        raise ValueError("Kloc must be a tensor [L, Hkv, B, T, d]")
    B, T = Kloc.shape[2], Kloc.shape[3]
    for t, nm in ((Kloc, "Kloc"), (Vloc, "Vloc")):
        _need(t, nm, torch.bfloat16, (L_, Hkv, B, T, d), Q.device)
    for t, nm, n in ((q_seq, "q_seq", nq), (q_pos, "q_pos", nq), (local_len, "local_len", B)):
        _need(t, nm, torch.int32, (n,), Q.device)
    return B, T


def merge_local(a, A_doc, Q, q_seq, q_pos, Kloc, Vloc, local_len, scale: Optional[float] = None, out=None,
                stream=None):
    """out [L,Hkv,G,nq,d] fp32: Eqs. (3.4)-(3.5) merge of (a, A_doc) with the
    exact causal attention over Kloc, Vloc [L,Hkv,B,T,d]."""
    dims, nq = dims_of(Q)
    _need(Q, "Q", torch.bfloat16)
    _need(a, "a", torch.float32, Q.shape[:4], Q.device)
    _need(A_doc, "A_doc", torch.float32, Q.shape, Q.device)
    B, T = _local_args(q_seq, q_pos, Kloc, Vloc, local_len, Q)
    if scale is None:
        scale = 1.0 / math.sqrt(dims.d)
    out = _out(out, "out", torch.float32, Q.shape, Q.device)
    st = lib().nectar_merge_local(dims, _ptr(a), _ptr(A_doc), _ptr(Q), nq, _ptr(q_seq), _ptr(q_pos), _ptr(Kloc),
                                  _ptr(Vloc), B, T, _ptr(local_len), float(scale), _ptr(out), _stream(stream))
    _check(st, "nectar_merge_local")
    return out


def decode_workspace_size(mods: ModuleSet, G: int, nq: int, d: int = 128) -> int:
    return int(lib().nectar_decode_workspace_size(Dims(mods.L, mods.Hkv, G, d), mods.c(), nq))


def decode(mods: ModuleSet, Q, q_seq, q_pos, Kloc, Vloc, local_len, scale: Optional[float] = None, out=None,
           workspace=None, stream=None):
    """Module forward + merge with local attention: out [L,Hkv,G,nq,d] fp32.
    workspace: uint8 CUDA tensor of decode_workspace_size(...) bytes, made
    here when None."""
    dims, nq = dims_of(Q)
    _need(Q, "Q", torch.bfloat16)
    _need_mods(mods, dims)
    B, T = _local_args(q_seq, q_pos, Kloc, Vloc, local_len, Q)
    if scale is None:
        scale = 1.0 / math.sqrt(dims.d)
    out = _out(out, "out", torch.float32, Q.shape, Q.device)
    workspace = _workspace(workspace, decode_workspace_size(mods, dims.G, nq, dims.d), Q.device)
    st = lib().nectar_decode(dims, mods.c(), _ptr(Q), nq, _ptr(q_seq), _ptr(q_pos), _ptr(Kloc), _ptr(Vloc), B, T,
                             _ptr(local_len), float(scale), _ptr(out), _ptr(workspace),
                             0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "nectar_decode")
    return out


def decode_layer_out(mods: ModuleSet, Q, q_seq, q_pos, Kloc, Vloc, local_len, scale: Optional[float] = None,
                     out=None, workspace=None, stream=None):
    """The decode as a base-model attention layer: bf16 out [L, nq, Hkv*G, d]
    (query head h*G + g), the fp32 result of decode() rounded to nearest."""
    dims, nq = dims_of(Q)
    _need(Q, "Q", torch.bfloat16)
    _need_mods(mods, dims)
    B, T = _local_args(q_seq, q_pos, Kloc, Vloc, local_len, Q)
    if scale is None:
        scale = 1.0 / math.sqrt(dims.d)
    out = _out(out, "out", torch.bfloat16, (dims.L, nq, dims.Hkv * dims.G, dims.d), Q.device)
    workspace = _workspace(workspace, int(lib().nectar_decode_layer_out_workspace_size(dims, mods.c(), nq)),
                           Q.device)
    st = lib().nectar_decode_layer_out(dims, mods.c(), _ptr(Q), nq, _ptr(q_seq), _ptr(q_pos), _ptr(Kloc),
                                       _ptr(Vloc), B, T, _ptr(local_len), float(scale), _ptr(out), _ptr(workspace),
                                       0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "nectar_decode_layer_out")
    return out


def quadrature_init(K, V, p: int, W=None, Z=None, stream=None):
    """Quadrature module rows (section 2.4) initialised to the first p rows of
    the cache: W, Z bf16 [L, Hkv, p, d] (made here when None)."""
    if not isinstance(K, torch.Tensor) or K.dim() != 4:
        raise ValueError("K must be a tensor [L, Hkv, n, d]")
    L_, Hkv, n, d = K.shape
    for t, nm in ((K, "K"), (V, "V")):
        _need(t, nm, torch.bfloat16, K.shape, K.device)
    if p < 0:
        raise ValueError(f"p = {p}: need 1 <= p <= n")
    W = _out(W, "W", torch.bfloat16, (L_, Hkv, p, d), K.device)
    Z = _out(Z, "Z", torch.bfloat16, (L_, Hkv, p, d), K.device)
    st = lib().nectar_quadrature_init(Dims(L_, Hkv, 1, d), _ptr(K), _ptr(V), n, p, _ptr(W), _ptr(Z),
                                      _stream(stream))
    _check(st, "nectar_quadrature_init")
    return W, Z


def quadrature_forward(W, Z, Q, scale: Optional[float] = None, a=None, A_theta=None, workspace=None, stream=None):
    """(a_theta [L,Hkv,G,nq], A_theta [L,Hkv,G,nq,d]) fp32 of the Quadrature
    module with rows W, Z bf16 [L, Hkv, p, d]."""
    dims, nq = dims_of(Q)
    p = _cache_args(W, Z, Q, dims)
    if scale is None:
        scale = 1.0 / math.sqrt(dims.d)
    a = _out(a, "a", torch.float32, Q.shape[:4], Q.device)
    A_theta = _out(A_theta, "A_theta", torch.float32, Q.shape, Q.device)
    workspace = _workspace(workspace, int(lib().nectar_quadrature_workspace_size(dims, p, nq)), Q.device)
    st = lib().nectar_quadrature_forward(dims, _ptr(W), _ptr(Z), p, _ptr(Q), nq, float(scale), _ptr(a),
                                         _ptr(A_theta), _ptr(workspace),
                                         0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "nectar_quadrature_forward")
    return a, A_theta


def fit_metrics(alpha, A, a, A_theta, Q, metrics=None, stream=None):
    """Per (l, h) [score MSE, target MSE, RTE term] (float64 [L, Hkv, 3]) of a
    module's (a, A_theta) against the exact (alpha, A); the RTE of Eq. (C.1)
    is metrics[..., 2].sum()."""
    dims, nq = dims_of(Q)
    _need(Q, "Q", torch.bfloat16)
    for t, nm in ((alpha, "alpha"), (a, "a")):
        _need(t, nm, torch.float32, Q.shape[:4], Q.device)
    for t, nm in ((A, "A"), (A_theta, "A_theta")):
        _need(t, nm, torch.float32, Q.shape, Q.device)
    metrics = _out(metrics, "metrics", torch.float64, (dims.L, dims.Hkv, 3), Q.device)
    st = lib().nectar_fit_metrics(dims, nq, _ptr(alpha), _ptr(A), _ptr(a), _ptr(A_theta), _ptr(Q), _ptr(metrics),
                                  _stream(stream))
    _check(st, "nectar_fit_metrics")
    return metrics


def device_error_flags(clear: bool = True) -> int:
    """Device error word (bit 0 wait timeout, 1 bad q_seq, 2 bad local_len).
    Synchronises the device."""
    v = ctypes.c_int32(0)
    _check(lib().nectar_device_error_flags(ctypes.byref(v), 1 if clear else 0), "nectar_device_error_flags")
    return int(v.value)


def check_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueue the library's bounded-wait self-check: a wait that nothing
    completes gives up after limit_us and sets bit 0 of the device error
    word (read it with device_error_flags)."""
    _check(lib().nectar_check_wait_timeout(int(limit_us), _stream(stream)), "nectar_check_wait_timeout")
