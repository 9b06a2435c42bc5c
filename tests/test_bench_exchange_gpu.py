"""bench.py's exchange across real ranks (--gpus N > 1), end to end, with two
ranks sharing this GPU: gloo carries the host-side collectives (the barriers
around the pull kernel, the all-to-alls of the NCCL path, the IPC handle
exchange), each rank maps the other's planes through CUDA IPC, and no kernel
waits on another. The line must report that the pull path and the all-to-all
path agree bit for bit on every rank."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("config,extra", [("decode", []), ("ulysses", ["--tokens", "4096"])])
def test_bench_exchange_two_ranks_on_one_gpu(config, extra):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--gpus", "2", "--steps", "3", "--warmup", "3", "--config", config] + extra
    env = {**os.environ, "CPLSE_BENCH_BACKEND": "gloo"}
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-4000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2 and rec["config"]["parallelism"] == "dcp2"
    assert rec["exchange"]["pull_equals_a2a"] is True
    assert rec["value"] > 0 and rec["roofline"]["bound"] == "nvlink"
    p50, p95 = rec["exchange"]["pull_rank_max_us_p50_p95"]
    assert 0 < p50 <= p95
    if config == "ulysses":
        assert rec["ulysses_exchange"]["pull_equals_nccl"] is True
