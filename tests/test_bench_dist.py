"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The benchmark runs one process per GPU with independent batches (weak scaling,
no data-path collective); its only collectives are barriers and the maximum of
the per-rank times.  These tests run that logic as two gloo ranks."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    from local_global_attention_b200 import configs as C
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    # every rank gets the maximum of the per-rank times
    t = bench.max_over_ranks(10.0 + rank, w)
    bench.barrier(w)
    wl = bench.rank_workload(C.VOL65K, rank)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": t, "seed": wl.seed, "shape": [wl.B, wl.H, wl.Z, wl.Y, wl.X]}, f)
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # max over ranks, seen by every rank
    assert all(r["max"] == 11.0 for r in res)
    # weak scaling: same shape, different batches
    assert res[0]["shape"] == res[1]["shape"]
    assert res[0]["seed"] != res[1]["seed"]


def test_whole_job_rate_counts_all_ranks():
    import bench
    # 131,072 tokens per rank, 4 ranks, slowest rank 2 ms
    assert bench.whole_job_rate(131072, 4, 2.0) == pytest.approx(131072 * 4 / 2e-3)


def test_reference_arm_only_on_rank_zero(monkeypatch):
    """Under torchrun the oracle arm runs on rank 0 alone; other ranks exit
    without work or output."""
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(workload="vol_32x32x64", packing="random", steps=1, warmup=3,
                              cpu_sample=64))()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""


def test_reference_arm_line_on_rank_zero(monkeypatch):
    """Rank 0 of the oracle arm prints one JSON line with the CUDA arm's metric,
    unit and config, the cpu_baseline it measured and a zero-copy e2e."""
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), dict(workload="tiny_8x8x8", packing="raster", steps=1, warmup=3,
                              cpu_sample=64))()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["value"] > 0
    assert (line["steps"], line["warmup"], line["n_gpus"]) == (1, 3, 1)
    assert line["config"] == bench.run_config(bench.workload("tiny_8x8x8"), "raster", 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT,
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_algorithmic_work_counts_terms_by_enumeration():
    """The roofline's numerator: bench.algorithmic_work's local and summary
    term counts (per-axis closed forms) against a direct enumeration over
    every query voxel, its clipped window and every block box."""
    import itertools

    import numpy as np

    import bench
    from local_global_attention_b200 import inputs as I
    wl = I.Workload(name="enum", B=1, H=1, d=12, Z=5, Y=7, X=9, window=(3, 5, 3),
                    block=(5, 7, 3))
    r = [(w - 1) // 2 for w in wl.window]
    dims = (wl.Z, wl.Y, wl.X)
    nbs = [n // b for n, b in zip(dims, wl.block)]
    local = summ = 0
    for c in itertools.product(*(range(n) for n in dims)):
        lo = [max(c[a] - r[a], 0) for a in range(3)]
        hi = [min(c[a] + r[a], dims[a] - 1) for a in range(3)]
        local += int(np.prod([hi[a] - lo[a] + 1 for a in range(3)]))
        for B in itertools.product(*(range(n) for n in nbs)):
            meets = all(B[a] * wl.block[a] <= hi[a] and (B[a] + 1) * wl.block[a] - 1 >= lo[a]
                        for a in range(3))
            summ += 0 if meets else 1
    w = bench.algorithmic_work(wl)
    assert w["local_flop"] == 4 * wl.d * local
    assert w["summary_flop"] == 4 * wl.d * summ
    assert w["bwd_flop"] == 10 * wl.d * (local + summ)
