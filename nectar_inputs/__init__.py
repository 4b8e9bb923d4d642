"""Seeded synthetic workloads for the Nectar hot path.

This module only draws random numbers and lays them out.  It holds none of
the method's arithmetic (no scores, no softmax, no MLP), so that both the
CUDA path and the CPU oracle can read the same inputs without sharing any
of the code that is being checked.

Shapes follow the workloads of "Nectar: Neural Estimation of
Cached-Token Attention via Regression" (Monteiro, Klein, Ablin, Cuturi):
a fixed n-token document cache K, V in R^{n x d} per (layer, KV-head) with
RoPE already applied (notes §2.1), GQA query heads that share one KV head
and one module pair (§2.1), module widths set by the capacity
rho = |theta| / (2 n d) (§2.5), and exact local (instruction / generated)
tokens after the document (§2.2).  The documents, trained modules and base
models of the paper are not available; every tensor here is synthetic.

Layouts (all contiguous, d innermost):
  K, V   bf16 [L][Hkv][n][d]            document cache, one per (l, h)
  Q      bf16 [L][Hkv][G][nq][d]        query head h' = h*G + g, token i
  Kloc, Vloc bf16 [L][Hkv][B][T][d]     local cache of every sequence
  q_seq, q_pos int32 [nq]               sequence and local position of token i
  local_len int32 [B]                   valid local tokens of each sequence
  modules: per layer, per net ("score", "target"), bf16 tensors with a
           leading Hkv axis:  U[k] [Hkv][H][H or d], V[k] [Hkv][H][d]
           (V[0] is None: layer 0 has no re-injection), b[k] [Hkv][H],
           Wout [Hkv][dout][H], c [Hkv][dout].
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, List, Optional, Sequence

import torch

D_HEAD = 128

# ---------------------------------------------------------------------------
# Presets.  Each is one of the workloads the Nectar pages measure on, reduced
# to the shapes that matter for the attention / module / merge path.
# ---------------------------------------------------------------------------
PRESETS: Dict[str, dict] = {
    # Toy single (layer, KV-head): 64 local tokens, each one a query token
    # for all G=4 query heads (256 query vectors), document n=4096, H=256.
    "toy": dict(L=1, Hkv=1, G=4, n=4096, B=1, T=64, nq=64, mode="prefill",
                H=256, key_scale=None, heavy=False, modules=True),
    # Qwen3-1.7B shape: 28 x 8 KV heads, GQA 2, n=32768, per-head key scale
    # U(0.5, 2), H=512, batch-1 decode after 512 local tokens.
    "qwen3_1p7b": dict(L=28, Hkv=8, G=2, n=32768, B=1, T=512, nq=1,
                       mode="decode", H=512, key_scale=(0.5, 2.0),
                       heavy=False, modules=True),
    # Qwen3-4B shape, regression-target generation: 36 x 8 KV heads, GQA 4,
    # n=61440, 4 heavy-hitter key directions (+6 logit), 1024 query tokens
    # x 4 query heads = 4096 query vectors per (l, h).  Exact (alpha, A) only.
    "qwen3_4b_targets": dict(L=36, Hkv=8, G=4, n=61440, B=0, T=0, nq=1024,
                             mode="targets", H=0, key_scale=None, heavy=True,
                             modules=False),
    # Qwen2.5-7B shape Nectar decode: 28 x 4 KV heads, GQA 7, n=131072,
    # H=768, 64 sequences of 256 local tokens, one new token each.
    "qwen25_7b_decode": dict(L=28, Hkv=4, G=7, n=131072, B=64, T=256, nq=64,
                             mode="decode", H=768, key_scale=None,
                             heavy=False, modules=True),
    # Llama-3.1-8B shape sweep: 32 x 8 KV heads, GQA 4, n=65536, 128 local
    # tokens, batch in {1, 16, 256}, rho in {1, 5, 10}% with non-uniform
    # per-layer widths (x1.5 on the first and last 4 layers).
    "llama8b_sweep": dict(L=32, Hkv=8, G=4, n=65536, B=16, T=128, nq=16,
                          mode="decode", H=None, rho=0.05, key_scale=None,
                          heavy=False, modules=True),
}

HEAVY_LOGIT = 6.0          # additive logit of a heavy-hitter key
N_HEAVY = 4                # heavy-hitter directions per (l, h)
BIAS_STD = 0.02            # module biases (the workloads do not fix them)


def _seed(*parts) -> int:
    """Stable 63-bit seed from a tuple of labels (independent of PYTHONHASHSEED)."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def module_params_per_head(H: int, d: int = D_HEAD, depth: int = 2) -> int:
    """Parameter count of one (score, target) pair with `depth` hidden layers
    of width H, input re-injection in every layer after the first, and a
    linear readout (1 output for the score net, d for the target net)."""
    hidden = H * d + H + (depth - 1) * (H * (d + H) + H)
    return 2 * hidden + (H + 1) + (d * H + d)


def capacity(H: int, n: int, d: int = D_HEAD, depth: int = 2) -> float:
    """rho = |theta| / (2 n d) for one (layer, KV-head)  (notes §2.5)."""
    return module_params_per_head(H, d, depth) / (2.0 * n * d)


def width_for_params(P: float, d: int = D_HEAD, depth: int = 2) -> float:
    """Real H with module_params_per_head(H) == P (depth 2: a quadratic)."""
    # params(H) = 2*depth_quadratic: collect a*H^2 + b*H + c
    a = 2.0 * (depth - 1)
    b = 2.0 * (d + 1 + (depth - 1) * (d + 1)) + 1 + d
    c = 1.0 + d
    if a == 0:
        return (P - c) / b
    return (-b + math.sqrt(b * b - 4 * a * (c - P))) / (2 * a)


def nonuniform_widths(rho: float, L: int, n: int, d: int = D_HEAD,
                      edge_layers: int = 4, edge_mult: float = 1.5,
                      multiple: int = 16) -> List[int]:
    """Per-layer widths for capacity rho with the first and last
    `edge_layers` layers given `edge_mult` x the parameters of the others,
    renormalised so that the total equals rho * 2nd * L (notes §2.5, and the
    layer-group capacity ablation of App. C.1).  Widths round to `multiple`."""
    mult = [edge_mult if (l < edge_layers or l >= L - edge_layers) else 1.0
            for l in range(L)]
    total = rho * 2.0 * n * d * L
    unit = total / sum(mult)
    out = []
    for m in mult:
        H = width_for_params(unit * m, d)
        out.append(max(multiple, int(round(H / multiple)) * multiple))
    return out


@dataclasses.dataclass
class Workload:
    name: str
    L: int
    Hkv: int
    G: int
    d: int
    n: int
    nq: int
    B: int
    T: int
    scale: float
    K: torch.Tensor
    V: torch.Tensor
    Q: torch.Tensor
    q_seq: Optional[torch.Tensor] = None
    q_pos: Optional[torch.Tensor] = None
    local_len: Optional[torch.Tensor] = None
    Kloc: Optional[torch.Tensor] = None
    Vloc: Optional[torch.Tensor] = None
    widths: Optional[List[int]] = None
    depth: int = 2
    modules: Optional[List[Dict[str, dict]]] = None
    meta: dict = dataclasses.field(default_factory=dict)

    @property
    def rows(self) -> int:
        """Query vectors per (layer, KV-head): G * nq."""
        return self.G * self.nq

    @property
    def heads(self) -> int:
        return self.L * self.Hkv


def _randn(shape, gen, device, dtype=torch.float32):
    return torch.randn(shape, generator=gen, device=device, dtype=dtype)


def _heavy_hitters(Kh: torch.Tensor, Qh: torch.Tensor, gen, device):
    """Plant N_HEAVY heavy-hitter keys in one (l, h) cache (in place, fp32).

    Directions u_1..u_4 are orthonormal; key j_i = HEAVY_LOGIT*sqrt(d)*u_i
    plus Gaussian noise projected off span(u); every query's component along
    each u_i is set to exactly 1.  A heavy key then scores
    HEAVY_LOGIT + N(0, ~1) against N(0, 1) for an ordinary key."""
    n, d = Kh.shape
    U, _ = torch.linalg.qr(_randn((d, N_HEAVY), gen, device))     # d x 4
    pos = torch.randint(1, n, (N_HEAVY - 1,), generator=gen, device=device)
    pos = torch.cat([torch.zeros(1, dtype=pos.dtype, device=device), pos])
    for i in range(N_HEAVY):
        z = Kh[pos[i]]
        z = z - U @ (U.T @ z)
        Kh[pos[i]] = HEAVY_LOGIT * math.sqrt(d) * U[:, i] + z
    # queries: replace the span(u) component by sum_i u_i
    Qh -= (Qh @ U) @ U.T
    Qh += U.sum(dim=1)
    return pos


def make_modules(L: int, Hkv: int, widths: Sequence[int], d: int, seed: int,
                 device, depth: int = 2) -> List[Dict[str, dict]]:
    """Random-init score and target nets for every (l, h): weights
    N(0, 1/fan_in), biases N(0, BIAS_STD^2), bf16."""
    mods = []
    for l in range(L):
        H = widths[l]
        layer = {}
        for net, dout in (("score", 1), ("target", d)):
            g = _gen(device, seed, "module", l, net)
            U, Vs, b = [], [], []
            for k in range(depth):
                fan_in = d if k == 0 else d + H
                std = 1.0 / math.sqrt(fan_in)
                U.append((_randn((Hkv, H, d if k == 0 else H), g, device) * std).to(torch.bfloat16))
                Vs.append(None if k == 0 else
                          (_randn((Hkv, H, d), g, device) * std).to(torch.bfloat16))
                b.append((_randn((Hkv, H), g, device) * BIAS_STD).to(torch.bfloat16))
            Wout = (_randn((Hkv, dout, H), g, device) / math.sqrt(H)).to(torch.bfloat16)
            c = (_randn((Hkv, dout), g, device) * BIAS_STD).to(torch.bfloat16)
            layer[net] = dict(U=U, V=Vs, b=b, Wout=Wout, c=c, H=H, dout=dout)
        mods.append(layer)
    return mods


def make_modules_general(L: int, Hkv: int, d: int, seed: int, device, depths: Sequence[int],
                         width_b: Sequence[int], width_s: Sequence[int],
                         width_t: Sequence[int]) -> List[Dict[str, dict]]:
    """Random-init module sets with a shared backbone: depths (D_b, D_s, D_t)
    of the backbone, score and target branches, per-layer widths of each.
    The backbone is D_b layers of the Eq. (3.6) recursion; each branch
    continues it from the backbone's last hidden state (its first layer sees
    q and that state), then its linear readout.  A layer that starts a chain
    (D_b = 0) sees only q: U [H][d], V None.  Weights N(0, 1/fan_in), biases
    N(0, BIAS_STD^2), bf16.  With D_b = 0 and equal widths the draws are
    those of make_modules."""
    Db, Ds, Dt = depths
    mods = []
    for l in range(L):
        layer = {}
        Hb = width_b[l] if Db > 0 else 0
        g = _gen(device, seed, "module", l, "backbone")
        U, Vs, b = [], [], []
        for k in range(Db):
            prev = 0 if k == 0 else Hb
            std = 1.0 / math.sqrt(d + prev)
            U.append((_randn((Hkv, Hb, prev if prev else d), g, device) * std).to(torch.bfloat16))
            Vs.append(None if prev == 0 else (_randn((Hkv, Hb, d), g, device) * std).to(torch.bfloat16))
            b.append((_randn((Hkv, Hb), g, device) * BIAS_STD).to(torch.bfloat16))
        layer["backbone"] = dict(U=U, V=Vs, b=b, H=Hb)
        for net, dout, D, Ws in (("score", 1, Ds, width_s), ("target", d, Dt, width_t)):
            H = Ws[l]
            g = _gen(device, seed, "module", l, net)
            U, Vs, b = [], [], []
            for k in range(D):
                prev = Hb if k == 0 else H
                std = 1.0 / math.sqrt(d + prev)
                U.append((_randn((Hkv, H, prev if prev else d), g, device) * std).to(torch.bfloat16))
                Vs.append(None if prev == 0 else (_randn((Hkv, H, d), g, device) * std).to(torch.bfloat16))
                b.append((_randn((Hkv, H), g, device) * BIAS_STD).to(torch.bfloat16))
            Wout = (_randn((Hkv, dout, H), g, device) / math.sqrt(H)).to(torch.bfloat16)
            c = (_randn((Hkv, dout), g, device) * BIAS_STD).to(torch.bfloat16)
            layer[net] = dict(U=U, V=Vs, b=b, Wout=Wout, c=c, H=H, dout=dout)
        mods.append(layer)
    return mods


def _module_widths(cfg: dict, L: int, n: int, d: int) -> List[int]:
    """Per-layer widths of a workload's modules: explicit, uniform H, or
    solved per layer from the capacity rho."""
    if "widths" in cfg:
        return list(cfg["widths"])
    if cfg.get("H"):
        return [int(cfg["H"])] * L
    return nonuniform_widths(cfg["rho"], L, n, d)


def workload_shape(name: str, **overrides) -> dict:
    """The sizes make_workload(name, **overrides) builds, without building
    anything: name, L, Hkv, G, d, n, B, T, nq, and the modules' per-layer
    widths (empty without modules) and depth."""
    cfg = dict(PRESETS[name])
    cfg.update(overrides)
    L, n = cfg["L"], cfg["n"]
    d = cfg.get("d", D_HEAD)
    nq = cfg["nq"]
    if cfg["mode"] == "decode":
        nq = cfg.get("nq", cfg["B"]) if "nq" in overrides else cfg["B"]
    with_modules = cfg.get("with_modules", cfg.get("modules", False))
    return dict(name=name, L=L, Hkv=cfg["Hkv"], G=cfg["G"], d=d, n=n, B=cfg["B"], T=cfg["T"], nq=nq,
                widths=_module_widths(cfg, L, n, d) if with_modules else [], depth=cfg.get("depth", 2))


def make_workload(name: str, *, seed: int = 0, device="cpu", **overrides) -> Workload:
    """Build a preset workload (optionally with overridden sizes).

    Overrides: any preset key (L, Hkv, G, n, B, T, nq, H, rho, ...), plus
    `widths` (explicit per-layer list) and `with_modules` / `with_local`."""
    cfg = dict(PRESETS[name])
    cfg.update(overrides)
    L, Hkv, G, n = cfg["L"], cfg["Hkv"], cfg["G"], cfg["n"]
    d = cfg.get("d", D_HEAD)
    mode = cfg["mode"]
    B, T, nq = cfg["B"], cfg["T"], cfg["nq"]
    if mode == "decode":
        nq = cfg.get("nq", B) if "nq" in overrides else B
    dev = torch.device(device)

    K = torch.empty((L, Hkv, n, d), dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    Q = torch.empty((L, Hkv, G, nq, d), dtype=torch.bfloat16, device=dev)
    heavy_pos = {}
    for l in range(L):
        for h in range(Hkv):
            g = _gen(dev, seed, "doc", l, h)
            Kh = _randn((n, d), g, dev)
            Vh = _randn((n, d), g, dev)
            Qh = _randn((G * nq, d), g, dev)
            if cfg.get("key_scale"):
                lo, hi = cfg["key_scale"]
                s = lo + (hi - lo) * torch.rand((), generator=g, device=dev)
                Kh *= s
            if cfg.get("heavy") and n > N_HEAVY:
                heavy_pos[(l, h)] = _heavy_hitters(Kh, Qh, g, dev).cpu()
            K[l, h] = Kh.to(torch.bfloat16)
            V[l, h] = Vh.to(torch.bfloat16)
            Q[l, h] = Qh.view(G, nq, d).to(torch.bfloat16)

    wl = Workload(name=name, L=L, Hkv=Hkv, G=G, d=d, n=n, nq=nq, B=B, T=T,
                  scale=1.0 / math.sqrt(d), K=K, V=V, Q=Q,
                  meta=dict(cfg=cfg, seed=seed, heavy_pos=heavy_pos))

    with_local = cfg.get("with_local", mode in ("decode", "prefill"))
    if with_local and B > 0 and T > 0:
        Kloc = torch.empty((L, Hkv, B, T, d), dtype=torch.bfloat16, device=dev)
        Vloc = torch.empty_like(Kloc)
        for l in range(L):
            g = _gen(dev, seed, "local", l)
            Kloc[l] = _randn((Hkv, B, T, d), g, dev).to(torch.bfloat16)
            Vloc[l] = _randn((Hkv, B, T, d), g, dev).to(torch.bfloat16)
        if "local_len" in cfg:
            local_len = torch.as_tensor(cfg["local_len"], dtype=torch.int32)
        else:
            local_len = torch.full((B,), T, dtype=torch.int32)
        if mode == "prefill":
            # every local token of sequence 0 queries (causal prefill)
            q_seq = torch.zeros(nq, dtype=torch.int32)
            q_pos = torch.arange(nq, dtype=torch.int32)
        else:
            # one new token per sequence, at the last local position
            q_seq = torch.arange(nq, dtype=torch.int32) % max(B, 1)
            q_pos = (local_len[q_seq.long()] - 1).clamp(min=0).to(torch.int32)
        if "q_seq" in cfg:
            q_seq = torch.as_tensor(cfg["q_seq"], dtype=torch.int32)
        if "q_pos" in cfg:
            q_pos = torch.as_tensor(cfg["q_pos"], dtype=torch.int32)
        wl.Kloc, wl.Vloc = Kloc, Vloc
        wl.q_seq, wl.q_pos, wl.local_len = q_seq.to(dev), q_pos.to(dev), local_len.to(dev)

    with_modules = cfg.get("with_modules", cfg.get("modules", False))
    if with_modules:
        widths = _module_widths(cfg, L, n, d)
        wl.widths = widths
        wl.depth = cfg.get("depth", 2)
        wl.modules = make_modules(L, Hkv, widths, d, seed, dev, wl.depth)
    return wl


def kv_cache_bytes(n: int, L: int, Hkv: int, d: int, bytes_per=2) -> int:
    """Footprint of a document KV cache: 2 n L H d numbers (notes §1)."""
    return 2 * n * L * Hkv * d * bytes_per
