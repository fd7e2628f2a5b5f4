"""The N > 1 host plumbing of bench.py on CPU: two gloo ranks (world size 2).

The path has no exchange step (every (sequence, head) is independent), so
bench.py --gpus N runs N replicas; what needs checking is the timing
reduction (max over ranks), the barrier, the whole-job value and the
reference arm's rank-0-only behaviour.  The GPU side is the same code with
the NCCL backend.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per_rank_ms = [3.0, 5.0][rank]
        m = bench.max_over_ranks(per_rank_ms, dist)
        bench.barrier(dist)
        v = bench.job_value(8192, world, m)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": m, "value": v}, f)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for g in got:
        assert g["max"] == 5.0                       # the slowest rank sets the time
        assert g["value"] == pytest.approx(2 * 8192 / 5e-3)


def test_reference_arm_prints_on_rank0_only():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                                       "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"],
                                      env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      cwd=ROOT, text=True))
    outs = [p.communicate(timeout=600) for p in procs]
    assert [p.returncode for p in procs] == [0, 0], [o[1][-2000:] for o in outs]
    line = json.loads(outs[0][0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert outs[1][0].strip() == ""
    # the contract's keys, and the reference-arm additions
    for key in ("metric", "unit", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["steps"] == 1 and line["warmup"] == 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "varlen8_h32_d128_resume"
    # rank 0 alone works: the value is one host's throughput, not scaled by N
    assert line["host"] == {"ranks_working": 1, "ranks_launched": 2}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
