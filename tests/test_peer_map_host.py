"""The peer mapping of the pull exchange decides as a group, on CPU: gloo
process groups of 2 ranks run PeerMap with fakes standing in for the IPC calls
(no GPU, nothing is mapped). When one rank fails to export or to map a peer's
buffer, every rank must raise PeerMapError at the same point, none may be left
waiting in a collective, and each must unmap what it had mapped."""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import lse_pack_stable_b200 as cp
        from lse_pack_stable_b200 import exchange as ex
        opened, closed = [], []

        def fake_export(t):
            if mode == "export_fails" and rank == 0:
                raise cp.CplseError(-6, "export refused (fake)")
            return b"rank%d-tensor%d" % (rank, t.numel())

        def fake_import(blob):
            if mode == "import_fails" and rank == 1:
                raise cp.CplseError(-6, "import refused (fake)")
            base = 4096 * (len(opened) + 1)
            opened.append(base)
            return base, base + 16

        def fake_close(base):
            closed.append(base)

        ex.ipc_export, ex.ipc_import, ex.ipc_close = fake_export, fake_import, fake_close
        tensors = [torch.zeros(8), torch.zeros(3)]
        try:
            pm = ex.PeerMap(tensors)
        except ex.PeerMapError as e:
            q.put((rank, "error", str(e), len(opened), sorted(closed) == sorted(opened)))
            return
        kinds = [[type(x).__name__ for x in pm.table(i)] for i in range(len(tensors))]
        addrs = [pm.table(i)[1 - rank].data_ptr() for i in range(len(tensors))]
        pm.close()
        q.put((rank, "ok", (kinds, addrs), len(opened), sorted(closed) == sorted(opened)))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "crash", repr(e), -1, False))
        raise
    finally:
        dist.destroy_process_group()


def _run(mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, *rest = q.get(timeout=120)
        got[r] = rest
    for p in procs:
        p.join(60)
    return got


def test_peer_map_all_ranks_succeed():
    got = _run("ok")
    for r in (0, 1):
        status, (kinds, addrs), n_opened, all_closed = got[r]
        assert status == "ok"
        own = ["Tensor", "_Plane"] if r == 0 else ["_Plane", "Tensor"]
        assert kinds == [own, own]
        assert addrs == [4096 + 16, 2 * 4096 + 16]     # base + the exported offset
        assert n_opened == 2 and all_closed


def test_peer_map_failed_import_is_everyone_s_error():
    got = _run("import_fails")
    assert [got[r][0] for r in (0, 1)] == ["error", "error"], got
    assert "this rank" in got[1][1] and "another rank" in got[0][1]
    assert got[0][2] == 2 and got[0][3], "rank 0 must unmap what it had mapped"
    assert got[1][2] == 0


def test_peer_map_failed_export_is_everyone_s_error():
    got = _run("export_fails")
    assert [got[r][0] for r in (0, 1)] == ["error", "error"], got
    assert all("rank(s) [0]" in got[r][1] for r in (0, 1))
    assert got[0][2] == 0 and got[1][2] == 0
