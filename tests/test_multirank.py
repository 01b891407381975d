"""The multi-rank host logic of bench.py on CPU: gloo ranks on 127.0.0.1.
The decode path needs no exchange between GPUs (replicas), so what spans
ranks is the timing: every rank's times are reduced by max, and the job's
rate counts the units of all ranks over that time."""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402

_RANK = r"""
import datetime, json, os, sys
import torch, torch.distributed as dist
sys.path.insert(0, os.environ["TQ_ROOT"])
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.25 * rank], world, torch.device("cpu"))
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "got": got}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_two_gloo_ranks():
    port = str(_free_port())
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=port, TQ_ROOT=str(ROOT))
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["got"] == [2.0, 10.0, 0.25]   # the slowest rank per entry


def test_whole_job_rate_counts_every_rank():
    assert bench.whole_job_rate(16 * 32768, 1, 0.25) == pytest.approx(16 * 32768 / 0.25e-3)
    assert bench.whole_job_rate(16 * 32768, 4, 0.25) == pytest.approx(4 * 16 * 32768 / 0.25e-3)


def test_reference_arm_under_torchrun_prints_one_line():
    """Rank 0 alone times the oracle and prints; the other rank exits 0."""
    port = str(_free_port())
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", port, str(ROOT / "bench.py"), "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
