"""The multi-rank (N > 1) side of bench.py, on CPU: world_size-2 process
groups over gloo.  The path runs replicas -- one independent stack per GPU, no
data exchange -- so what the ranks share is the timing protocol (a barrier on
both sides of the timed loop, the slowest rank's time, the whole-job rate)
and the reference arm's rule that rank 0 alone runs and prints."""
import datetime
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


def _worker(rank, world, port, values, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier()
        slowest = bench._max_over_ranks(values[rank])
        bench._barrier()
        rate = bench.whole_job_rate(world, 1, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_slowest_rank_and_whole_job_rate_over_gloo(tmp_path):
    """Every rank gets the slowest rank's step time (max over ranks), and the
    whole-job rate is N x the per-rank units over that time."""
    world = 2
    values = [2.5, 4.0]   # per-rank step times (ms)
    mp.start_processes(_worker, args=(world, _free_port(), values, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["slowest"] == 4.0
        assert g["rate"] == pytest.approx(world * 1 / 4.0e-3)


def test_whole_job_rate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_rate(1, 1, 1.0) == pytest.approx(1000.0)
    # doubling the replicas at the same step time doubles the job's rate
    assert bench.whole_job_rate(2, 1, 1.0) == pytest.approx(2 * bench.whole_job_rate(1, 1, 1.0))
    # the job is as slow as its slowest rank
    assert bench.whole_job_rate(8, 4, 2.0) == pytest.approx(8 * 4 / 2.0e-3)


def test_reference_arm_rank0_prints_one_line_other_ranks_exit_silently():
    """Under torchrun with N = 2 the reference arm (the CPU oracle) runs on
    rank 0 only; the other rank exits 0 without work or output."""
    outs = {}
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                            "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=300,
                           cwd=ROOT)
        assert r.returncode == 0, r.stderr[-2000:]
        outs[rank] = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
