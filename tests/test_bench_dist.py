"""bench.py's multi-process host path on CPU: two ranks over gloo.

The hot path has no exchange step (every sequence is independent), so N GPUs
run N replicas; the only cross-rank traffic is the barrier around the timed
region and the max over ranks of the measured time.  These tests run that
plumbing as two CPU processes (gloo, 127.0.0.1), and the reference arm, which
only rank 0 runs and prints.
"""
import importlib.util
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))


def _max_worker(rank, world, port, out_dir):
    _env(rank, world, port)
    bench = _bench()

    class Args:
        pass

    w, r, _ = bench.dist_setup(Args())
    try:
        bench.barrier(w)
        got = bench.max_over_ranks(1.5 + 10.0 * r, w)   # rank 1 is the slow one
        with open(os.path.join(out_dir, f"max{r}.json"), "w") as f:
            json.dump({"world": w, "rank": r, "max": got}, f)
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def _reference_worker(rank, world, port, out_dir):
    _env(rank, world, port)
    bench = _bench()
    path = os.path.join(out_dir, f"ref{rank}.out")
    with open(path, "w") as f:
        sys.stdout = f
        rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1",
                         "--warmup", "1", "--workload", "tiny_f32", "--ref-seconds", "0.5"])
        sys.stdout.flush()
    with open(os.path.join(out_dir, f"rc{rank}"), "w") as f:
        f.write(str(rc))


def test_max_over_ranks_and_barrier_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_max_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        d = json.load(open(tmp_path / f"max{r}.json"))
        assert d["world"] == 2 and d["rank"] == r
        assert d["max"] == pytest.approx(11.5)   # every rank sees the slowest rank's time


def test_reference_arm_prints_once_on_rank_zero(tmp_path):
    port = _free_port()
    mp.start_processes(_reference_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    assert (tmp_path / "rc0").read_text() == "0" and (tmp_path / "rc1").read_text() == "0"
    assert (tmp_path / "ref1.out").read_text().strip() == ""      # rank 1 does no work
    lines = [l for l in (tmp_path / "ref0.out").read_text().splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["parallelism"] == "replicas2"
