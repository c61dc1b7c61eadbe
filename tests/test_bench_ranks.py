"""The bench's N > 1 host logic on CPU: two ranks launched the way the
multi-GPU bench is launched (torchrun, loopback rendezvous), gloo instead of
NCCL.  Checks the max-over-ranks timing, the whole-job throughput and that the
reference arm prints exactly one line, from rank 0."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun(args, timeout=240):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port())] + args
    env = dict(os.environ, OMP_NUM_THREADS="2")
    return subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout, env=env)


def json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_two_ranks_time_is_the_slowest_rank():
    r = torchrun([os.path.join("tests", "ranks_worker.py")])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    res = lines[0]
    assert res["world"] == 2
    assert sorted(p["rank"] for p in res["per_rank"]) == [0, 1]
    assert all(p["slowest"] == 15.0 for p in res["per_rank"])  # every rank agrees on the max
    assert res["value"] == pytest.approx(2 * 1e12 / 15e-3 / 1e12)  # both ranks' work / slowest time


def test_reference_arm_two_ranks_prints_one_line():
    r = torchrun(["bench.py", "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
                  "--warmup", "0", "--cpu-tokens", "16"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
