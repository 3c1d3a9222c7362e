"""Multi-rank paths of bench.py, on the CPU with gloo ranks (world size 2).

The GPU arm runs one independent replica per GPU and needs two things from the ranks: the job
time is the slowest rank's time (every rank must agree on it), and the job value counts the
work of all ranks.  The reference arm (the CPU oracle) runs on rank 0 only and prints one line;
the other ranks exit 0 without work.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = bench.max_over_ranks(100.0 + 25.0 * rank, torch.device("cpu"))
        value = bench.job_value(world, 8, 1000, 10, elapsed)
        # the e2e leg's host-buffer mode: every rank takes the smallest mode any rank can afford
        mode = bench.all_ranks_min(2 - rank, torch.device("cpu"))
        with open(os.path.join(out, "rank%d.json" % rank), "w") as f:
            json.dump({"elapsed": elapsed, "value": value, "mode": mode}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    for g in got:
        assert g["elapsed"] == 125.0  # the slower rank's time, on every rank
        assert abs(g["value"] - world * 8 * 1000 * 10 / 0.125) < 1e-6
        assert g["mode"] == 1  # both ranks agree on the mode the poorer rank can afford


def test_e2e_host_mode():
    import bench
    W, n = 8, 10 ** 9
    assert bench.e2e_host_mode(W, n, None, 1) == 2
    assert bench.e2e_host_mode(W, n, 196 << 30, 1) == 2  # 36 GB of pinned buffers for one rank
    assert bench.e2e_host_mode(W, n, 196 << 30, 8) == 1  # eight ranks share the host: 8 GB each
    assert bench.e2e_host_mode(W, n, 20 << 30, 8) == 0


def test_reference_arm_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "gauss64k"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
