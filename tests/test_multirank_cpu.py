"""The multi-rank host logic of the benchmark (replicas, weak scaling) on
CPU ranks over gloo, world size 2: per-rank batches differ, the step time is
the max over ranks on every rank, and the value counts all ranks' tokens.
The reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as wl  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(times[rank], world)
        wr = bench.rank_workload(wl.TINY, rank)
        x = wl.gen_router_inputs(wr)["x_f32"]
        np.save(os.path.join(out_dir, f"x{rank}.npy"), x)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{ms_max!r} {bench.aggregate_tokens_per_s(world, wr.T, ms_max)!r}")
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_aggregate(tmp_path):
    world, times = 2, [1.25, 3.5]
    tmp.spawn(_rank_main, args=(world, _free_port(), times, str(tmp_path)), nprocs=world,
              join=True)
    res = [open(tmp_path / f"r{r}.txt").read().split() for r in range(world)]
    for ms, val in res:
        assert float(ms) == max(times)
        assert float(val) == pytest.approx(world * wl.TINY.T / (max(times) / 1e3))
    x0, x1 = (np.load(tmp_path / f"x{r}.npy") for r in range(world))
    assert x0.shape == x1.shape and not np.array_equal(x0, x1)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(2.0, 1) == 2.0
    assert bench.rank_workload(wl.TINY, 0) == wl.TINY
    assert bench.aggregate_tokens_per_s(1, 1000, 2.0) == pytest.approx(5e5)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_reference_arm_line_has_the_contract_keys():
    """Rank 0 of the reference arm (the fp64 oracle on the host) prints one
    JSON line with the benchmark's keys, its own arithmetic and an e2e
    object equal to its value."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 3
    assert d["config"]["workload"] == wl.V3_FULL.name
    assert d["config"]["router_precision"].startswith("fp64")
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1


def test_gpus_flag_without_launcher_starts_one_rank_per_gpu():
    """`bench.py --gpus 2` with no launcher starts the two ranks itself (the
    environment torchrun would give them); rank 0 alone prints one line and
    it reports n_gpus = 2.  The reference arm needs no GPU, so this runs on
    CPU."""
    import json
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"


@pytest.mark.parametrize("impl", ["ours", "reference"])
def test_gpus_flag_disagreeing_with_launcher_fails(impl):
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", impl,
                        "--gpus", "4", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert p.returncode != 0 and "WORLD_SIZE" in p.stderr
    assert p.stdout.strip() == ""
