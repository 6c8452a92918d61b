"""The N > 1 plumbing of bench.py on the CPU: two ranks over gloo.

The path has no exchange step (each (b, h) is independent), so N GPUs run N
independent replicas and the only collectives are the timing ones: a barrier
around the timed region and the maximum of the step time over ranks.  These
tests run that plumbing with world_size 2 on gloo, without a GPU.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench

    bench.barrier(world)
    # each rank reports a different step time; every rank must see the largest
    m = bench.allmax(1.5 + rank, world, torch.device("cpu"))
    with open(os.path.join(outdir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(m))
    bench.barrier(world)
    dist.destroy_process_group()


def test_step_time_is_the_maximum_over_two_ranks(tmp_path):
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    got = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(2)]
    assert got == [2.5, 2.5]


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
