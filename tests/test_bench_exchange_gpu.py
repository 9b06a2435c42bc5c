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


def _fallback_worker(rank, world, port, q, extra):
    import contextlib
    import io
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world), CPLSE_BENCH_BACKEND="gloo")
    try:
        import bench
        import lse_pack_stable_b200 as cp
        from lse_pack_stable_b200 import exchange as ex
        real_import = ex.ipc_import

        def import_refused_on_rank_1(blob):     # the failure is made on the host
            if rank == 1:
                raise cp.CplseError(-6, "peer mapping refused (test)")
            return real_import(blob)
        ex.ipc_import = import_refused_on_rank_1
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            rc = bench.run_ours(bench.parse(["--gpus", "2", "--steps", "3", "--warmup", "3"]
                                            + extra))
        q.put((rank, rc, out.getvalue()))
    except Exception as e:  # noqa: BLE001
        q.put((rank, -1, repr(e)))
        raise


@pytest.mark.parametrize("extra", [["--config", "decode"],
                                   ["--config", "ulysses", "--tokens", "4096"]])
def test_bench_exchange_falls_back_to_nccl_path_when_mapping_fails(extra):
    """One rank cannot map its peer's planes: every rank learns it at the same
    point, no rank hangs, and the line times the all-to-all path and says why
    (on Ulysses the load/store transforms say they were unavailable too)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fallback_worker, args=(r, 2, port, q, extra)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        r, rc, text = q.get(timeout=600)
        got[r] = (rc, text)
    for p in procs:
        p.join(120)
    assert got[0][0] == 0 and got[1][0] == 0, got
    lines = [l for l in got[0][1].splitlines() if l.startswith("{")]
    assert len(lines) == 1, got[0][1][-2000:]
    rec = json.loads(lines[0])
    assert rec["exchange"]["timed_path"] == "a2a"
    assert "another rank" in rec["exchange"]["pull_unavailable"]
    assert rec["exchange"]["pull_equals_a2a"] is None
    assert rec["value"] > 0 and "NCCL" in rec["roofline"]["kernel"]
    assert not [l for l in got[1][1].splitlines() if l.startswith("{")]   # rank 0 prints
    if "ulysses" in extra:
        assert "another rank" in rec["ulysses_exchange"]["unavailable"]
