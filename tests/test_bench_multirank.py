"""The multi-rank plumbing of bench.py, run as two gloo ranks on the CPU.

The data path has no collective (every rank runs its own layer); what crosses
ranks is the timing: a barrier on both sides of the timed region, the
slowest rank's time, and one JSON line printed by rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_body(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    class Args:
        gpus = world
    w, r, local = bench.dist_setup(Args())
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    # each rank reports a different step time; all must agree on the slowest
    t = bench.max_over_ranks(0.5 + 0.25 * rank, w)
    v = bench.whole_job_value(w, 1e12, t)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"t": t, "v": v}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path):
    world = 2
    mp.start_processes(_rank_body, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    slowest = 0.5 + 0.25 * (world - 1)
    for g in got:
        assert g["t"] == pytest.approx(slowest)
        # two ranks of 1 TFLOP each over the slowest rank's time
        assert g["v"] == pytest.approx(world * 1.0 / slowest)


def test_whole_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_value(1, 2e12, 1.0) == pytest.approx(2.0)
    assert bench.whole_job_value(8, 2e12, 1.0) == pytest.approx(16.0)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
