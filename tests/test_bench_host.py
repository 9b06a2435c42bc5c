"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks timing reduce, the whole-job throughput, and the reference arm
under torchrun (rank 0 alone prints one JSON line, the other rank exits 0)."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.reduce_max([1.0 + rank, 10.0 - rank, 3.5], world, "cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [2.0, 10.0, 3.5]


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 1 GB per step x 10 steps in 1 s of (max) device time
    assert bench.job_throughput(2, 1e9, 10, 1000.0) == pytest.approx(20.0)
    assert bench.reduce_max([3.0, 1.0], 1, "cpu") == [3.0, 1.0]


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "1", "--config", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["unit"] == "GB/s"
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0


def test_ab_decision_rule():
    """The paired A/B's rule: positive needs >= 75 % of blocks for the
    candidate AND a median improvement above max(1 %, 2 x noise floor)."""
    sys.path.insert(0, ROOT)
    import bench
    null = [0.004, -0.003, 0.002, -0.006]            # noise floor = median |e| = 0.0035
    pos = bench.ab_decision([0.2, 0.21, 0.19, 0.2, 0.22, 0.18, 0.2, 0.2], null)
    assert pos["verdict"] == "positive" and pos["blocks_favouring_candidate"] == "8/8"
    assert pos["noise_floor"] == pytest.approx(0.0035) and pos["threshold"] == pytest.approx(0.01)
    # 6/8 blocks (75 %) favour the candidate, median effect 1.5 % > 1 %: positive
    assert bench.ab_decision([0.02, 0.02, 0.015, 0.015, 0.02, 0.015, -0.01, -0.01],
                             null)["verdict"] == "positive"
    # 5/8 favour the candidate: neutral however large the effect
    assert bench.ab_decision([0.3, 0.3, 0.3, 0.3, 0.3, -0.1, -0.1, -0.1], null)["verdict"] == "neutral"
    # a noisy floor raises the threshold: 3 % improvement against a 2 % floor (4 % bar)
    assert bench.ab_decision([0.03] * 8, [0.02, -0.02, 0.02, -0.02])["verdict"] == "neutral"
    # the mirror image is a regression
    assert bench.ab_decision([-0.05] * 8, null)["verdict"] == "regression"


def test_rotation_policy_is_a_function_of_the_workload():
    """Both arms print the same config, so the L2 note cannot depend on the device."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    assert bench.rotation_sets(synth.CONFIGS["stress"]) == 1
    assert bench.rotation_sets(synth.CONFIGS["mla"]) == 1
    n = bench.rotation_sets(synth.CONFIGS["decode"])
    assert n >= 2 and n * synth.CONFIGS["decode"].fused_bytes() >= 3 * bench.L2_BYTES
    a = bench.config_block(synth.CONFIGS["decode"], 1)
    assert a == bench.config_block(synth.CONFIGS["decode"], 1) and "l2" in a
