"""The multi-rank logic of bench.py on CPU: world-size-2 gloo ranks agree on
the max time over ranks, the whole-job value counts every rank's work over
that time, and the reference arm does no work on ranks other than 0."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [12.5, 20.0][rank]
    ms_max = bench.reduce_max(local_ms, world, torch.device("cpu"))
    value = bench.whole_job_tflops(1e12, world, 10, ms_max)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"ms_max": ms_max, "value": value}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value(tmp_path):
    import socket
    with socket.socket() as sock:  # a port that is free right now
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    assert res[0]["ms_max"] == res[1]["ms_max"] == 20.0
    # 2 ranks x 10 steps x 1 TFLOP over the slowest rank's 20 ms
    assert res[0]["value"] == pytest.approx(2 * 10 * 1.0 / 0.020)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
