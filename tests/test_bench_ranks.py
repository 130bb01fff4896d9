"""bench.py's multi-rank plumbing on CPU, with two gloo ranks.

`bench.py --gpus N` runs one process per GPU: every rank meets the others at a
barrier before and after its timed region and the job's time is the maximum
over ranks. These tests run that plumbing with two CPU processes over gloo on
127.0.0.1: the barrier and the max-over-ranks reduction, and the reference arm
under the torch.distributed launcher, where rank 0 alone prints the JSON line
and the other rank exits 0 without work. `bench.py --gpus 2` without a launcher
starts the two ranks itself, and a launcher whose rank count differs from --gpus
is refused.
"""
import json
import os
import socket
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    r, w = bench.init_ranks(types.SimpleNamespace(impl="reference"))
    assert (r, w) == (rank, world)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    got = bench.max_over_ranks(1.0 + 3.5 * rank, w)  # ranks offer 1.0 and 4.5
    bench.barrier(w)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(got))


def test_barrier_and_max_over_ranks_with_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for rank in range(2):
        assert float((tmp_path / f"rank{rank}.txt").read_text()) == 4.5


def test_max_over_ranks_is_identity_for_one_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.25, 1) == 7.25


def test_reference_arm_under_the_launcher_with_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "tiny_decode", "--ref-budget-s", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["config"]["workload"] == "tiny_decode"
    assert res["value"] > 0 and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0


def test_bench_starts_its_own_ranks_without_a_launcher():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "3", "--workload", "tiny_decode", "--ref-budget-s", "1"]
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["OMP_NUM_THREADS"] = "2"
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["config"]["parallelism"] == "replicas x2"


def test_bench_refuses_a_rank_count_other_than_gpus():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "3", "--steps", "1",
           "--warmup", "3", "--workload", "tiny_decode"]
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode != 0 and "--gpus 3" in p.stderr
