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


def torchrun(args, timeout=240, nproc=2):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(nproc),
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


def test_reference_arm_one_process_line_has_the_contract_keys():
    # launched as the driver launches N = 1 (no torchrun)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                        "--warmup", "1", "--cpu-tokens", "16"], cwd=ROOT, capture_output=True, text=True,
                       timeout=240, env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    line = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 1
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["config"]["workload"] == "tiny"
    assert line["cpu_baseline"]["value"] == line["value"] and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
