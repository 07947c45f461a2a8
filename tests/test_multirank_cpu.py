"""Two-rank host logic of bench.py on CPU (gloo): the max-over-ranks timing
reduction, the barrier, and the reference arm, which rank 0 alone runs and prints."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(float(10 * (rank + 1)), world, torch.device("cpu"))
        bench.barrier(world)
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1",
                             "--warmup", "3", "--workload", "tiny", "--ref-seconds", "0.05"])
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": m, "rc": rc, "stdout": buf.getvalue()}, f)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_ranks_max_and_reference_arm(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["max"] == 20.0 and r1["max"] == 20.0
    assert r0["rc"] == 0 and r1["rc"] == 0
    assert r1["stdout"].strip() == ""  # only rank 0 runs and prints the reference arm
    line = json.loads(r0["stdout"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tok/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
