"""The N > 1 path of bench.py on CPU: two ranks over the gloo backend.

Every rank times its own steps; the bench reduces the times with a max over
ranks (all ranks take part) and reports the whole job's rate, every rank's
units over that time (weak scaling).  The reference arm under torchrun runs
on rank 0 alone and the other ranks exit 0 without work.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", init_method="env://", timeout=datetime.timedelta(seconds=60))
local_ms = [4.0, 7.5][rank]
bench.barrier(dist, world)
m = bench.max_over_ranks(local_ms, dist, world, "cpu")
rate = bench.whole_job_rate(1e9, world, m)
dist.destroy_process_group()
print(json.dumps({{"rank": rank, "max_ms": m, "rate": rate}}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_max_time_and_sum_the_units():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_SCRIPT.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["max_ms"] == 7.5  # both ranks see the slower rank's time
        assert abs(o["rate"] - 2 * 1e9 / 7.5e-3) < 1e-3 * o["rate"]  # both ranks' units over it


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "single_256x128", "--gpus", "2", "--steps", "1",
           "--warmup", "1", "--ref-step-seconds", "0.2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
