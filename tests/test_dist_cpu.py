"""Two-rank CPU checks of the multi-process paths (gloo, world size 2).

The layer runs as independent data-parallel replicas (one rank per GPU, no
data-path collective); these tests cover the host side of that on CPU: the
rendezvous, the barrier, the max-over-ranks of the timed duration, the per-rank
batches, and the reference arm printing exactly one line from rank 0.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun(args, timeout=240):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", "--master-port=%d" % free_port()] + args
    env = dict(os.environ, OMP_NUM_THREADS="1")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def test_replica_plumbing_two_ranks(tmp_path):
    r = torchrun([os.path.join(ROOT, "tests", "dist_worker.py"), str(tmp_path)])
    assert r.returncode == 0, r.stderr[-3000:]
    res = [json.load(open(tmp_path / ("rank_%d.json" % i))) for i in range(2)]
    for i, d in enumerate(res):
        assert d["rank"] == i and d["world"] == 2
        assert d["max"] == pytest.approx(13.5)          # the slowest replica's time
        assert d["all"] == res[0]["all"]
    a, b = res[0]["all"]
    assert a["w"] == b["w"]                              # same layer weights
    assert a["x"] != b["x"]                              # a batch of its own per replica


def test_reference_arm_prints_once(tmp_path):
    r = torchrun([os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--config", "1",
                  "--steps", "1", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
