"""bench.py's multi-rank bookkeeping on CPU with gloo, world size 2: the
step time is the max over ranks and the throughput counts every rank's
units over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    assert bench.dist_env() == (world, rank, rank)
    ms = [10.0, 25.0][rank]                     # rank 1 is the slow one
    mx = bench.reduce_max(ms)
    value = bench.aggregate(448, mx, steps=20)  # 448 query vectors per rank-step
    bench.barrier()
    out[rank] = (mx, value)
    dist.destroy_process_group()


def test_bench_aggregation_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        mx, value = out[r]
        assert mx == 25.0
        assert value == pytest.approx(2 * 448 * 20 / 0.025)


def test_bench_single_process_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.aggregate(448, 10.0, steps=10) == pytest.approx(448 * 10 / 0.010)


@pytest.mark.parametrize("name,over", [
    ("toy", {}),
    ("qwen3_1p7b", dict(L=3, n=256)),
    ("qwen3_4b_targets", dict(L=2, n=256, nq=8)),
    ("qwen25_7b_decode", dict(L=2, n=256, B=3, T=8)),
    ("llama8b_sweep", dict(L=10, n=1024, B=2, T=8)),          # widths solved per layer from rho
])
def test_workload_shape_is_what_make_workload_builds(name, over):
    from nectar_inputs import make_workload, workload_shape
    import bench
    s = workload_shape(name, **over)
    wl = make_workload(name, **over)
    for k in ("L", "Hkv", "G", "d", "n", "B", "T", "nq"):
        assert s[k] == getattr(wl, k), k
    assert s["widths"] == (wl.widths or [])
    assert bench.describe_shape(s) == bench.describe(wl)


def test_reference_sample_is_layer_0_of_the_full_workload():
    """With widths solved from rho, layer 0 of a 32-layer set is wider than a
    one-layer set of the same capacity: the reference arm's one-layer sample
    must take the full workload's layer-0 width."""
    from nectar_inputs import workload_shape
    full = workload_shape("llama8b_sweep")
    alone = workload_shape("llama8b_sweep", L=1)
    assert full["widths"][0] > alone["widths"][0]


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the keys of the bench contract."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "toy",
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["config"]["workload"].startswith("toy: L=1 ")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
