"""Benchmark of the Nectar hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3_1p7b]

One step = the whole hot path over one decode batch of the workload:
(i) exact cached-token attention (alpha, A) over the document (Eq. (3.1))
and the Nectar decode -- (ii) the score / target MLPs (Eq. (3.6)) fused with
(iii) the merge with exact causal local attention (Eqs. (3.4)-(3.5)).  The
metric is query vectors (layer x query head x token) per second through the
step; the dominant kernel is (i), which is HBM-bound, so its roofline is
reported as achieved / measured HBM bandwidth.

Multi-GPU: one process per GPU under torchrun; every rank runs an
independent replica (the path has no exchange step), value = all ranks'
queries / max-over-ranks time, scaling "weak".

--impl reference times the CPU oracle (oracle/, plain C in fp64) on the
host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nectar_inputs import PRESETS, make_workload, workload_shape  # noqa: E402

METRIC = "Nectar decode queries/s & exact (α,A) HBM GB/s at 1 B200; % of roofline"
UNIT = "queries/s"


def load_sustained(default):
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return default


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# distributed helpers (also exercised by the gloo tests)
# ---------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max over ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(units_per_rank: float, max_ms: float, steps: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    total_units = reduce_sum(units_per_rank * steps)
    return total_units / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples every 20 ms from a little before the timed region
    to a little after it; summary() keeps the samples whose timestamp falls
    inside [mark_start(), mark_end()] (host clock), and says how many."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # the samples go to $NECTAR_CLOCKS_DIR (default: the system temp directory)
        out_dir = os.environ.get("NECTAR_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_gpu{gpu_index}.csv")
        self.t_start = self.t_end = None

    def mark_start(self):
        self.t_start = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        try:
            rows = [ln.split(",") for ln in open(self.path).read().strip().splitlines() if ln.strip()]
        except Exception:
            rows = []
        import datetime
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        parsed = []
        for r in rows:
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                parsed.append((ts, float(r[2]), float(r[3]), [v.strip().lower() == "active" for v in r[6:10]]))
            except Exception:
                pass
        inside = [x for x in parsed
                  if self.t_start is not None and self.t_end is not None and self.t_start <= x[0] <= self.t_end]
        use = inside if inside else parsed
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "samples_in_timed_region": 0}
        reasons = sorted({nm for x in use for nm, on in zip(names, x[3]) if on})
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": use[-1][2], "reasons": reasons,
                "samples": len(parsed), "samples_in_timed_region": len(inside),
                "window": "timed region" if inside else "around the timed region (no sample inside it)"}


# ---------------------------------------------------------------------------
# workload bookkeeping
# ---------------------------------------------------------------------------
def describe(wl):
    return describe_shape(dict(name=wl.name, L=wl.L, Hkv=wl.Hkv, G=wl.G, d=wl.d, n=wl.n, B=wl.B, T=wl.T, nq=wl.nq,
                               widths=wl.widths or [], depth=wl.depth))


def describe_shape(s: dict) -> str:
    H = sorted(set(s["widths"]))
    return (f"{s['name']}: L={s['L']} Hkv={s['Hkv']} G={s['G']} d={s['d']} n={s['n']} B={s['B']} T={s['T']} "
            f"nq={s['nq']} H={H[0] if len(H) == 1 else H} depth={s['depth']}")


def queries_per_step(wl) -> int:
    return wl.L * wl.Hkv * wl.G * wl.nq


def attn_bytes(wl) -> int:
    """Algorithmic bytes of (i): K and V once per (l, h), Q in, alpha and A out."""
    heads, rows = wl.heads, wl.rows
    return heads * (4 * wl.n * wl.d + rows * 2 * wl.d + rows * 4 * (wl.d + 1))


def attn_flops(wl) -> int:
    """FLOPs of (i): q.k and p.v, 2 d each, for every (key, row) of every head."""
    return wl.heads * wl.rows * wl.n * 4 * wl.d


def decode_flops(wl) -> int:
    """FLOPs of the fused decode: 2 per module weight per row, plus local q.k
    and p.v over the visible tokens."""
    params = sum(wl.Hkv * (2 * H * H + 645 * H + 129) if wl.depth == 2 else 0 for H in wl.widths)
    vis = (torch.minimum(wl.q_pos.long().cpu() + 1, wl.local_len.long().cpu()[wl.q_seq.long().cpu()])).clamp(min=0)
    return 2 * params * wl.G * wl.nq + wl.heads * wl.G * int(vis.sum()) * 4 * wl.d


def decode_bytes(wl, weight_bytes: int) -> int:
    """Algorithmic bytes of the fused decode: module weights, the visible local
    K/V of every sequence, Q in, out."""
    vis = (wl.local_len.long().clamp(max=wl.T)).sum().item()
    return weight_bytes + wl.heads * vis * 4 * wl.d + wl.heads * wl.rows * (2 + 4) * wl.d


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def run_ours(args):
    import long_context_attention_split_b200 as nx
    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, peak_kind = load_peaks()
    tc_peak_sust = load_sustained(tc_peak)

    over = workload_overrides(args)
    wl = make_workload(args.workload, seed=args.seed + rank, device=dev, **over)
    has_decode = wl.modules is not None and wl.Kloc is not None
    mods = nx.pack_modules(wl.modules, wl.widths, wl.depth, wl.Hkv, wl.G, device=dev) if has_decode else None
    Q = wl.Q
    alpha = torch.empty(Q.shape[:4], dtype=torch.float32, device=dev)
    A = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    out = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    wsb = nx.cache_attn_workspace_size(wl.L, wl.Hkv, wl.G, wl.n, wl.nq)
    work = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    local_args = (wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len) if has_decode else None
    dwork = None
    if has_decode:
        dwork = torch.empty(nx.decode_workspace_size(mods, wl.G, wl.nq), dtype=torch.uint8, device=dev)
    # (i): main kernel + combine; decode: one launch + its merge, or with
    # >= 64 rows per KV head the local kernel, one GEMM per hidden layer and the readout
    if not has_decode:
        dec_launches = 0
    elif wl.rows >= 64:
        dec_launches = 1 + wl.depth + 1
    else:
        dec_launches = 2
    launches_per_step = 2 + dec_launches

    ev_a0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_a1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_d1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def step(i=None):
        if i is not None:
            ev_a0[i].record(stream)
        nx.cache_attn_lse(wl.K, wl.V, Q, alpha=alpha, A=A, workspace=work, stream=stream)
        if i is not None:
            ev_a1[i].record(stream)
        if has_decode:
            nx.decode(mods, Q, *local_args, out=out, workspace=dwork, stream=stream)
        if i is not None:
            ev_d1[i].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    flags = nx.device_error_flags(clear=True)

    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        barrier(dev)
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        clk.mark_start()
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
        barrier(dev)
    total_ms = t0.elapsed_time(t1)
    max_ms = reduce_max(total_ms, dev)
    attn_ms = [ev_a0[i].elapsed_time(ev_a1[i]) for i in range(args.steps)]
    dec_ms = [ev_a1[i].elapsed_time(ev_d1[i]) for i in range(args.steps)]
    attn_avg = sum(attn_ms) / len(attn_ms)
    dec_avg = sum(dec_ms) / len(dec_ms)
    flags |= nx.device_error_flags(clear=True)

    qps = queries_per_step(wl)
    value = aggregate(qps, max_ms, args.steps)
    ab = attn_bytes(wl)
    af = attn_flops(wl)
    db = decode_bytes(wl, mods.bytes) if has_decode else 0
    # dominant kernel: exact attention; HBM-bound below the ridge point
    # (query rows per KV head = FLOP per byte of K/V), tensor-bound above
    tensor_bound = wl.rows > tc_peak * 1e12 / (hbm_peak * 1e9)
    long_step = attn_avg > 10.0
    tc_use = tc_peak_sust if long_step else tc_peak
    if tensor_bound:
        achieved = af / (attn_avg / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_use,
                "peak_kind": f"{peak_kind} bf16 {'sustained' if long_step else 'burst'}",
                "unit": "TFLOP/s", "frac": achieved / tc_use, "alg_flops_per_launch": af,
                "alg_bytes_per_launch": ab, "hbm_GBps": ab / (attn_avg / 1e3) / 1e9}
    else:
        achieved = ab / (attn_avg / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "peak_kind": f"{peak_kind} copy",
                "unit": "GB/s", "frac": achieved / hbm_peak, "alg_bytes_per_launch": ab}

    # ---- the same step as L per-layer calls captured in one CUDA graph ----
    pp = parts(wl, attn_avg, dec_avg, ab, db, qps, hbm_peak, tc_peak, has_decode)
    exact_roof_us = max(ab / (hbm_peak * 1e9), af / (tc_peak * 1e12)) * 1e6
    dec_roof_us = pp.get("decode_roofline_us_full", 0.0)
    per_layer = per_layer_graph(wl, mods, Q, alpha, A, out, has_decode, dev, args,
                                roof_us={"step": exact_roof_us + dec_roof_us, "exact": exact_roof_us,
                                         "decode": dec_roof_us})
    nextr = next_rows(wl, mods, alpha, A, has_decode, dev, hbm_peak, tc_peak) if args.next_rows else None

    # ---- end to end through the public API with host buffers ----
    pin = lambda t: t.cpu().pin_memory()
    meta = (wl.q_seq, wl.q_pos, wl.local_len) if has_decode else ()
    h_in = [pin(Q)] + [pin(t) for t in meta]
    d_in = [torch.empty_like(Q)] + [torch.empty_like(t) for t in meta]
    d_out = [alpha, A] + ([out] if has_decode else [])
    h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in d_out]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)

    def e2e_step():
        for d, h in zip(d_in, h_in):
            d.copy_(h, non_blocking=True)
        nx.cache_attn_lse(wl.K, wl.V, d_in[0], alpha=alpha, A=A, workspace=work, stream=stream)
        if has_decode:
            nx.decode(mods, d_in[0], d_in[1], d_in[2], wl.Kloc, wl.Vloc, d_in[3], out=out, workspace=dwork,
                      stream=stream)
        for h, d in zip(h_out, d_out):
            h.copy_(d, non_blocking=True)

    e2e_value = None
    if not args.no_e2e:
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        barrier(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_max = reduce_max(e0.elapsed_time(e1), dev)
        e2e_value = aggregate(qps, e2e_max, args.steps)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        torch.cuda.synchronize(dev)
        gpu_out = {"alpha": alpha, "A": A, "out": out if has_decode else None}
        cpu = cpu_baseline(wl, budget_s=args.cpu_budget, gpu_out=gpu_out)

    if rank == 0:
        traffic = traffic_from_profile(args.workload)
        line = {
            "metric": METRIC,
            "value": value,
            "unit": UNIT,
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": max_ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                "workload": describe(wl),
                "global_batch": wl.B * ws,
                "seq_len": wl.n,
                "parallelism": f"replicas{ws}",
                "queries_per_step_per_gpu": qps,
                "l2": l2_note(ab),
            },
            "parts": dict(pp, per_layer_graph=per_layer, **({"next_rows": nextr} if nextr else {})),
            "roofline": dict(kernel=("cache_attn_tc+combine" if wl.rows > 8 else "cache_attn_split+combine")
                             + " (exact alpha, A)", traffic=traffic, **roof),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "device_error_flags": flags,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def parts(wl, attn_ms, dec_ms, ab, db, qps, hbm_peak, tc_peak, has_decode):
    out = {"exact_attn_ms": attn_ms, "exact_attn_GBps": ab / (attn_ms / 1e3) / 1e9,
           "exact_attn_TFLOPs": attn_flops(wl) / (attn_ms / 1e3) / 1e12,
           "exact_attn_queries_per_s": qps / (attn_ms / 1e3)}
    if has_decode:
        wbytes = db - wl.heads * (wl.local_len.long().clamp(max=wl.T)).sum().item() * 4 * wl.d \
            - wl.heads * wl.rows * 6 * wl.d
        dflops = decode_flops(wl)
        t = dec_ms / 1e3
        out.update({
            "decode_ms": dec_ms,
            "decode_queries_per_s": qps / t,
            "decode_alg_bytes": db,
            "decode_GBps": db / t / 1e9,
            "decode_flops": dflops,
            # full form: weights + local K/V bytes at HBM vs FLOPs at the tensor peak
            "decode_roofline_us_full": max(db / (hbm_peak * 1e9), dflops / (tc_peak * 1e12)) * 1e6,
            # weights-or-FLOPs form (module weights only)
            "decode_roofline_us_weights": max(wbytes / (hbm_peak * 1e9), dflops / (tc_peak * 1e12)) * 1e6,
        })
        out["decode_frac_full"] = out["decode_roofline_us_full"] / (dec_ms * 1e3)
        out["decode_frac_weights_form"] = out["decode_roofline_us_weights"] / (dec_ms * 1e3)
    return out


def _timed(fn, iters=10, warm=3):
    """Device time (ms) per call of fn() on the current stream: `iters` calls
    back to back between two CUDA events, so that the host's launch work
    overlaps the device's instead of sitting inside the timed region."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def next_rows(wl, mods, alpha, A, has_decode, dev, hbm_peak, tc_peak) -> dict:
    """The rows after the hot path, each on this workload's shapes, timed
    alone (inputs larger than L2 unless noted):
      quadrature: the Quadrature module forward at p = 10% of n;
      fit_metrics: score / target MSE and RTE over this step's targets;
      layer_out_decode: the decode as a base-model attention layer (bf16,
        layer layout);
      backbone_decode: the decode with a (2, 1, 2) module set (backbone,
        score, target depths) of this workload's widths."""
    import long_context_attention_split_b200 as nx
    from nectar_inputs import make_modules_general
    res = {}
    p = max(1, int(round(0.10 * wl.n)))
    W, Z = nx.quadrature_init(wl.K, wl.V, p)
    qa = torch.empty(wl.Q.shape[:4], dtype=torch.float32, device=dev)
    qA = torch.empty(wl.Q.shape, dtype=torch.float32, device=dev)
    qws = torch.empty(max(int(nx.lib().nectar_quadrature_workspace_size(nx.Dims(wl.L, wl.Hkv, wl.G, 128), p, wl.nq)),
                          16), dtype=torch.uint8, device=dev)
    t = _timed(lambda: nx.quadrature_forward(W, Z, wl.Q, a=qa, A_theta=qA, workspace=qws))
    # exact attention over p keys: bytes as (i) with n = p, FLOPs 4 p d per query row
    qbytes = 4 * p * 128 * wl.heads + wl.heads * wl.rows * (256 + 4 * 129)
    qflops = 4 * p * 128 * wl.heads * wl.rows
    q_roof_us = max(qbytes / (hbm_peak * 1e9), qflops / (tc_peak * 1e12)) * 1e6
    res["quadrature"] = {"p": p, "ms": t, "GBps": qbytes / (t / 1e3) / 1e9, "TFLOPs": qflops / (t / 1e3) / 1e12,
                         "bound": "hbm" if qbytes / (hbm_peak * 1e9) >= qflops / (tc_peak * 1e12) else "tensor",
                         "roofline_us": q_roof_us, "frac": q_roof_us / (t * 1e3), "alg_bytes": qbytes}
    del W, Z, qa, qA, qws
    # fit metrics: against the module's outputs, or -- for a workload without
    # modules (regression targets) -- against the targets shifted by 0.1 as
    # stand-in module outputs (the kernel reads the same bytes either way)
    if has_decode:
        mws = torch.empty(max(nx.module_workspace_size(mods, wl.G, wl.nq), 16), dtype=torch.uint8, device=dev)
        a, At = nx.module_forward(mods, wl.Q, workspace=mws)
    else:
        mws = None
        a, At = alpha + 0.1, A + 0.1
    met = torch.empty(wl.L, wl.Hkv, 3, dtype=torch.float64, device=dev)
    t = _timed(lambda: nx.fit_metrics(alpha, A, a, At, wl.Q, metrics=met))
    fbytes = wl.heads * wl.rows * (4 + 512 + 4 + 512 + 256)
    res["fit_metrics"] = {"ms": t, "GBps": fbytes / (t / 1e3) / 1e9,
                          "frac_hbm": fbytes / (t / 1e3) / 1e9 / hbm_peak, "alg_bytes": fbytes,
                          "l2": "inputs smaller than L2" if fbytes < 126e6 else "inputs larger than L2"}
    del a, At, mws
    if has_decode:
        # f1: the decode written as a base-model attention layer, bf16 in the
        # layer layout [L][nq][Hkv*G][d]; bytes as the fused decode's with a
        # 2-byte output
        lo = torch.empty((wl.L, wl.nq, wl.Hkv * wl.G, wl.d), dtype=torch.bfloat16, device=dev)
        lws_bytes = int(nx.lib().nectar_decode_layer_out_workspace_size(nx.Dims(wl.L, wl.Hkv, wl.G, wl.d), mods.c(),
                                                                         wl.nq))
        lws = torch.empty(max(lws_bytes, 16), dtype=torch.uint8, device=dev)
        largs = (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
        t = _timed(lambda: nx.decode_layer_out(mods, *largs, out=lo, workspace=lws))
        lbytes = decode_bytes(wl, mods.bytes) - wl.heads * wl.rows * 2 * wl.d
        l_roof_us = max(lbytes / (hbm_peak * 1e9), decode_flops(wl) / (tc_peak * 1e12)) * 1e6
        res["layer_out_decode"] = {"ms": t, "alg_bytes": lbytes, "roofline_us": l_roof_us,
                                   "frac": l_roof_us / (t * 1e3)}
        del lo, lws
        widths = list(wl.widths)
        gm = make_modules_general(wl.L, wl.Hkv, 128, 1, dev, (2, 1, 2), widths, widths, widths)
        arch = nx.Arch((2, 1, 2), widths, widths, widths)
        ms = nx.pack_modules_arch(gm, arch, wl.Hkv, wl.G, device=dev)
        params = sum(t.numel() for layer in gm for part in layer.values()
                     for key in ("U", "V", "b") for t in part[key] if t is not None) + \
            sum(layer[n][k].numel() for layer in gm for n in ("score", "target") for k in ("Wout", "c"))
        out = torch.empty(wl.Q.shape, dtype=torch.float32, device=dev)
        dws = torch.empty(nx.decode_workspace_size(ms, wl.G, wl.nq), dtype=torch.uint8, device=dev)
        args = (wl.Q, wl.q_seq, wl.q_pos, wl.Kloc, wl.Vloc, wl.local_len)
        t = _timed(lambda: nx.decode(ms, *args, out=out, workspace=dws))
        dbytes = decode_bytes(wl, 2 * params)           # bf16 weights + visible local K/V + Q + out
        classic = sum(wl.Hkv * (2 * H * H + 645 * H + 129) for H in wl.widths) if wl.depth == 2 else 0
        dflops = decode_flops(wl) - 2 * classic * wl.G * wl.nq + 2 * params * wl.G * wl.nq
        roof_us = max(dbytes / (hbm_peak * 1e9), dflops / (tc_peak * 1e12)) * 1e6
        res["backbone_decode"] = {"depths": [2, 1, 2], "ms": t, "params": params, "alg_bytes": dbytes,
                                  "roofline_us": roof_us, "frac": roof_us / (t * 1e3)}
    return res


def workload_overrides(args) -> dict:
    over = {}
    if args.layers:
        over["L"] = args.layers
    if args.batch:
        over["B"] = args.batch
    if args.rho:
        over["rho"] = args.rho
    if args.width:
        over["H"] = args.width
    return over


def l2_note(attn_bytes: float) -> str:
    if attn_bytes > 2 * 126e6:
        return f"inputs larger than L2 (document K/V {attn_bytes / 1e9:.2f} GB streamed every step)"
    return f"inputs of {attn_bytes / 1e6:.1f} MB fit in L2 (parity-size workload, not a bandwidth measurement)"


def per_layer_graph(wl, mods, Q, alpha, A, out, has_decode, dev, args, roof_us=None):
    """ms per step when the step is issued as L per-layer calls captured in
    one CUDA graph and replayed -- the form a model that runs layer after
    layer gives -- and the same for each half alone; None when the workload
    has one layer.  Four forms of the whole step, each with the
    dependencies a model that runs its layers in turn has (layer l + 1's
    query depends on layer l's decode output):
      `ms_per_step`: the decodes are the model's chain, on one stream; the
        exact attention of layer l (regression targets, which no later layer
        reads) starts on a second stream once layer l's query exists, i.e.
        after the decode of layer l - 1, and the step ends when both
        streams have;
      `beside_ms_per_step`: each layer's decode on a second stream beside
        its exact attention, the next layer after both;
      `serial_ms_per_step`: exact attention, then the decode, on one stream;
      `grouped4_ms_per_step`: as `ms_per_step`, but the exact attention
        runs for 4 layers at a time, once the last of their queries exists
        (not per-layer exact calls: the targets of a layer are ready up to
        3 layers later).
    roof_us: {"step": .., "exact": .., "decode": ..} roofline times (us) of
    the whole step and its halves, for the fractions."""
    if wl.L < 2:
        return None
    import long_context_attention_split_b200 as nx
    try:
        s = torch.cuda.Stream(dev)
        s2 = torch.cuda.Stream(dev)
        ws = torch.empty(max(nx.cache_attn_workspace_size(1, wl.Hkv, wl.G, wl.n, wl.nq), 16), dtype=torch.uint8,
                         device=dev)
        wsg = torch.empty(max(max(nx.cache_attn_workspace_size(k, wl.Hkv, wl.G, wl.n, wl.nq) for k in (1, 4)), 16),
                          dtype=torch.uint8, device=dev)
        lmods = [mods.layer(l) for l in range(wl.L)] if has_decode else None
        dws = torch.empty(max(max(nx.decode_workspace_size(m, wl.G, wl.nq) for m in lmods) if has_decode else 16, 16),
                          dtype=torch.uint8, device=dev)

        evs = [(torch.cuda.Event(), torch.cuda.Event()) for _ in range(wl.L)]
        end_b = torch.cuda.Event()

        def issue(exact=True, decode=True, beside=False, pipelined=False, group=1):
            if pipelined and exact and decode and has_decode:
                for l in range(wl.L):
                    sl = slice(l, l + 1)
                    q_ready = evs[l][0]
                    q_ready.record(s)            # after the decode of layer l - 1 (the step's start for l = 0)
                    if (l + 1) % group == 0 or l + 1 == wl.L:
                        gs = slice(l - l % group, l + 1)
                        s2.wait_event(q_ready)
                        nx.cache_attn_lse(wl.K[gs], wl.V[gs], Q[gs], alpha=alpha[gs], A=A[gs], workspace=wsg,
                                          stream=s2)
                    nx.decode(lmods[l], Q[sl], wl.q_seq, wl.q_pos, wl.Kloc[sl], wl.Vloc[sl], wl.local_len,
                              out=out[sl], workspace=dws, stream=s)
                end_b.record(s2)
                s.wait_event(end_b)
                return
            for l in range(wl.L):
                sl = slice(l, l + 1)
                if beside and exact and decode and has_decode:
                    # the exact attention first: issued after the decode, its
                    # CTAs waited behind the decode's (1.18 against 1.09 ms
                    # per step on Qwen3-1.7B)
                    fork, join = evs[l]
                    fork.record(s)
                    s2.wait_event(fork)
                    nx.cache_attn_lse(wl.K[sl], wl.V[sl], Q[sl], alpha=alpha[sl], A=A[sl], workspace=ws, stream=s)
                    nx.decode(lmods[l], Q[sl], wl.q_seq, wl.q_pos, wl.Kloc[sl], wl.Vloc[sl], wl.local_len,
                              out=out[sl], workspace=dws, stream=s2)
                    join.record(s2)
                    s.wait_event(join)
                    continue
                if exact:
                    nx.cache_attn_lse(wl.K[sl], wl.V[sl], Q[sl], alpha=alpha[sl], A=A[sl], workspace=ws, stream=s)
                if decode and has_decode:
                    nx.decode(lmods[l], Q[sl], wl.q_seq, wl.q_pos, wl.Kloc[sl], wl.Vloc[sl], wl.local_len,
                              out=out[sl], workspace=dws, stream=s)

        def timed(**kw):
            s.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(s):
                issue(**kw)             # first calls outside the capture (device setup)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
                issue(**kw)
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(s):
                e0.record(s)
                for _ in range(args.steps):
                    g.replay()
                e1.record(s)
            torch.cuda.synchronize(dev)
            del g
            return e0.elapsed_time(e1) / args.steps

        if has_decode:
            res = {"ms_per_step": timed(pipelined=True), "calls_per_step": wl.L * 2,
                   "beside_ms_per_step": timed(beside=True), "serial_ms_per_step": timed(),
                   "grouped4_ms_per_step": timed(pipelined=True, group=4)}
        else:
            res = {"ms_per_step": timed(), "calls_per_step": wl.L}
        res["exact_ms"] = timed(decode=False)
        if has_decode:
            res["decode_ms"] = timed(exact=False)
        if roof_us:
            res["frac_step"] = roof_us["step"] / (res["ms_per_step"] * 1e3)
            res["frac_exact"] = roof_us["exact"] / (res["exact_ms"] * 1e3)
            if has_decode:
                res["frac_decode_full"] = roof_us["decode"] / (res["decode_ms"] * 1e3)
        return res
    except Exception as ex:  # report, do not fail the bench line
        return {"error": f"{type(ex).__name__}: {ex}"[:200]}


# sources of the exact-attention kernels whose DRAM counters profiles/ records
_SPLIT_SOURCES = ("attn_decode.cu", "common.cuh", "ptx.cuh")


def split_sources_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in _SPLIT_SOURCES:
        with open(os.path.join(ROOT, "long_context_attention_split_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload: str):
    """DRAM bytes per full launch of the dominant kernel, read from the ncu
    summary in profiles/ (lines `dram_bytes_per_launch: B` and
    `sources_digest: X`); None when absent or when the kernel sources have
    changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"cache_attn_split_{workload}.md")
    try:
        with open(path) as f:
            text = f.read()
    except OSError:
        return None
    import re
    mb = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    md = re.search(r"sources_digest:\s*([0-9a-f]+)", text)
    if not mb or not md or md.group(1) != split_sources_digest():
        return None
    return int(mb.group(1))


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------
def _oracle_sample(wl, layers, keep=None):
    """One pass of the whole path on the oracle for the given layers (all
    their KV heads, the tokens kept in the host view).  Returns query
    vectors processed; with keep (a dict) also leaves the outputs there:
    alpha [H, rows], A [H, rows, d], out [H, rows, d] (H = layers x Hkv)."""
    import numpy as np
    import oracle
    H = len(layers) * wl.Hkv
    K = wl.K[layers].reshape(H, wl.n, wl.d)
    V = wl.V[layers].reshape(H, wl.n, wl.d)
    Q = wl.Q[layers].reshape(H, wl.rows, wl.d)
    alpha, A = oracle.cache_attn(K, V, Q, wl.scale)
    if keep is not None:
        keep.update(alpha=alpha, A=A)
    if wl.modules is None:
        return H * wl.rows
    sel = [(l, h) for l in layers for h in range(wl.Hkv)]
    a, At = oracle.module_forward(wl, sel)
    a = np.stack([a[k] for k in sel])
    At = np.stack([At[k] for k in sel])
    out = oracle.merge_local(a, At, Q, wl.q_seq, wl.q_pos, wl.Kloc[layers].reshape(H, wl.B, wl.T, wl.d),
                             wl.Vloc[layers].reshape(H, wl.B, wl.T, wl.d), wl.local_len, wl.scale)
    if keep is not None:
        keep.update(out=out, a=a, At=At)
    return H * wl.rows


def _sample_parity(wl, host, layers, ref, gpu_out) -> dict:
    """Max errors of the timed step's GPU outputs on the oracle sample's
    heads (layers `layers` of the workload, the host view's tokens), with
    the tolerances the parity tests use: alpha 1e-3 absolute, A 2e-3 of
    max|V|, the decode's out within the fused-decode bound (MLP 1e-2
    relative carried through the merge)."""
    import numpy as np
    idx = torch.tensor(layers)
    nq = host.nq

    def rows(t):          # [L, Hkv, G, nq, ...] -> [H, G * nq, ...] of the sample's layers and tokens
        t = t[idx.to(t.device)][:, :, :, :nq].cpu().numpy()
        return t.reshape(len(layers) * wl.Hkv, wl.G * nq, *t.shape[4:])

    res = {"heads": len(layers) * wl.Hkv, "layers": layers, "tokens": nq}
    vmax = float(host.V.float().abs().max())
    res["alpha_max_err"] = float(np.abs(rows(gpu_out["alpha"]) - ref["alpha"]).max())
    res["A_max_err"] = float(np.abs(rows(gpu_out["A"]) - ref["A"]).max())
    res["alpha_tol"] = 1e-3
    res["A_tol"] = 2e-3 * vmax
    ok = res["alpha_max_err"] <= res["alpha_tol"] and res["A_max_err"] <= res["A_tol"]
    if gpu_out.get("out") is not None and "out" in ref:
        a, At, o = ref["a"], ref["At"], ref["out"]
        vl = max(float(host.Vloc.float().abs().max()), float(np.abs(At).max()))
        bound = 1e-2 * np.abs(a).max() * (np.abs(At).max() + np.abs(o).max()) + 1e-2 * np.abs(At).max() + 2e-3 * vl
        res["out_max_err"] = float(np.abs(rows(gpu_out["out"]) - o).max())
        res["out_tol"] = float(bound)
        ok = ok and res["out_max_err"] <= res["out_tol"]
    res["pass"] = bool(ok)
    return res


def cpu_baseline(wl, budget_s=12.0, layers_per_sample=1, gpu_out=None):
    """The oracle timed on the host cores on a bounded sample of the
    workload (layer 0, all its KV heads).  With gpu_out (the timed step's
    alpha, A and out on the device) the sample's oracle outputs, and those
    of one more untimed pass over the last layer, also give the agreement of
    the step's GPU outputs on those heads ("parity")."""
    import oracle
    oracle.build()
    cores = oracle.num_threads()
    # host copies of what one sample touches: layer 0, and at most enough
    # tokens that one pass stays around a second
    layers = list(range(min(layers_per_sample, wl.L)))
    host = _host_view(wl, layers, token_cap=_token_cap(wl))
    t0 = time.perf_counter()
    done = 0
    samples = 0
    first = {}
    while True:
        done += _oracle_sample(host, list(range(len(layers))), keep=first if samples == 0 else None)
        samples += 1
        if time.perf_counter() - t0 > budget_s or samples >= 400:
            break
    dt = time.perf_counter() - t0
    # the same sample on one thread, for a quarter of the budget
    oracle.set_threads(1)
    try:
        t1 = time.perf_counter()
        done1 = samples1 = 0
        while True:
            done1 += _oracle_sample(host, list(range(len(layers))))
            samples1 += 1
            if time.perf_counter() - t1 > budget_s / 4 or samples1 >= 100:
                break
        dt1 = time.perf_counter() - t1
    finally:
        oracle.set_threads(cores)
    res = {"value": done / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
           "value_1core": done1 / dt1, "cpu_model": cpu_model(),
           "sample": f"{samples} pass(es) of the whole path over layer(s) {layers} "
                     f"({len(layers) * wl.Hkv} of {wl.heads} KV heads, {host.nq} of {wl.nq} tokens x {wl.G} "
                     f"query heads), {dt:.1f} s on {cores} threads; queries/s = query vectors done / time; "
                     f"value_1core: {samples1} pass(es) in {dt1:.1f} s on one thread"}
    if gpu_out is not None:
        par = [_sample_parity(wl, host, layers, first, gpu_out)]
        if wl.L > 1:
            last = [wl.L - 1]
            hl = _host_view(wl, last, token_cap=_token_cap(wl))
            ref = {}
            _oracle_sample(hl, [0], keep=ref)
            par.append(_sample_parity(wl, hl, last, ref, gpu_out))
        res["parity"] = par
    return res


def cpu_model() -> str:
    """The host CPU's model name, as the kernel reports it."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _token_cap(wl) -> int:
    """Tokens per sample so that the exact part of one pass is ~1e9 MACs."""
    per_token = wl.Hkv * wl.G * wl.n * wl.d * 3
    return max(1, min(wl.nq, int(1e9 // max(per_token, 1))))


class _HostWL:
    pass


def _host_view(wl, layers, token_cap=None):
    """CPU copy of the workload restricted to `layers` (renumbered 0..) and
    to the first `token_cap` query tokens."""
    h = _HostWL()
    for k in ("name", "Hkv", "G", "d", "n", "B", "T", "scale", "depth"):
        setattr(h, k, getattr(wl, k))
    nq = wl.nq if token_cap is None else min(token_cap, wl.nq)
    h.nq = nq
    h.L = len(layers)
    h.rows = wl.G * nq
    h.heads = h.L * wl.Hkv
    idx = torch.tensor(layers)
    h.K = wl.K[idx.to(wl.K.device)].cpu()
    h.V = wl.V[idx.to(wl.V.device)].cpu()
    h.Q = wl.Q[idx.to(wl.Q.device)][:, :, :, :nq].contiguous().cpu()
    h.modules = None
    h.widths = None
    if wl.Kloc is None or wl.modules is None:
        return h
    h.Kloc = wl.Kloc[idx.to(wl.Kloc.device)].cpu()
    h.Vloc = wl.Vloc[idx.to(wl.Vloc.device)].cpu()
    h.q_seq, h.q_pos, h.local_len = wl.q_seq[:nq].cpu(), wl.q_pos[:nq].cpu(), wl.local_len.cpu()
    h.widths = [wl.widths[l] for l in layers]
    h.modules = []
    for l in layers:
        layer = {}
        for net, p in wl.modules[l].items():
            layer[net] = {k: ([x.cpu() if x is not None else None for x in v] if isinstance(v, list)
                              else (v.cpu() if torch.is_tensor(v) else v)) for k, v in p.items()}
        h.modules.append(layer)
    return h


def run_reference(args):
    """The CPU oracle, as it stands, on the host's cores: each step is one
    pass of the whole path over layer 0 (all KV heads, all query rows) of the
    workload -- a bounded sample of the GPU arm's step."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    oracle.build()
    # layer 0 of the full workload: its module width is the full workload's
    # (widths solved per layer from rho depend on L)
    full = workload_shape(args.workload, **workload_overrides(args))
    over = dict(workload_overrides(args), L=1)
    if full["widths"]:
        over["widths"] = full["widths"][:1]
    wl = make_workload(args.workload, seed=args.seed, device="cpu", **over)
    host = _host_view(wl, [0], token_cap=_token_cap(wl))
    cores = oracle.num_threads()
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += _oracle_sample(host, [0])
    dt = time.perf_counter() - t0
    value = done / dt
    sample = (f"each step = the whole path over layer 0 of {full['L']} ({wl.Hkv} KV heads, {host.nq} of {wl.nq} "
              f"tokens x {wl.G} query heads) of {args.workload}")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": describe_shape(full), "global_batch": full["B"] * ws, "seq_len": full["n"],
                   "parallelism": f"{cores} host threads",
                   "queries_per_step_per_gpu": full["L"] * full["Hkv"] * full["G"] * full["nq"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3_1p7b", choices=sorted(PRESETS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--next-rows", action="store_true",
                    help="also time the Quadrature module, the fit metrics and a decode with a shared backbone")
    ap.add_argument("--batch", type=int, default=0, help="decode batch B (llama8b_sweep: 1, 16, 256)")
    ap.add_argument("--rho", type=float, default=0.0, help="module capacity (llama8b_sweep: 0.01, 0.05, 0.10)")
    ap.add_argument("--width", type=int, default=0,
                    help="module hidden width H for every layer (qwen25_7b_decode at rho = 10 %%: 1152)")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only the first LAYERS layers (small cases for profiling; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
