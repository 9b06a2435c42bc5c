"""The exchange across real ranks, host side, on CPU: gloo process groups of 2
and 3 ranks run the package's all-to-all exchange (its packet buffers, the
equal-split all-to-all of both regions, the hand-off to the combine) with the
float64 oracle standing in for the pack and the combine kernels. Each rank's
result must equal, bit for bit, destination `rank` of the oracle's own
single-process chain pack -> permute -> combine over all W planes."""
from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(W):
    import synth
    return synth.Workload("x%d" % W, W=W, T=6 * W, H=4 * W, D=16, dtype="bf16", seed=5 + W,
                          o_sigma=1.0, max_sigma=4.0, sum_dist=(synth.UNIFORM, 1.0, 100.0),
                          p_invalid=0.1, p_token_invalid=0.1)


def _oracle_pack(orc, fmt_unused=None):
    """cp_pack_lse_rank's contract, by the oracle: one plane, W destinations."""
    def pack(o, smax, ssum, W, scatter_dim, pkt_o, pkt_lse):
        on = o.view(torch.int16).numpy().view(np.uint16)
        planes = np.broadcast_to(on, (W,) + on.shape)          # plane 0 is this rank's
        mp_ = np.broadcast_to(smax.numpy(), (W,) + tuple(smax.shape))
        sp_ = np.broadcast_to(ssum.numpy(), (W,) + tuple(ssum.shape))
        pk, l32, _ = orc.pack(planes, mp_, sp_, scatter_dim)
        pkt_o.view(torch.int16).numpy()[...] = pk[0].view(np.int16)
        pkt_lse.numpy()[...] = l32[0]
    return pack


def _oracle_combine(orc, fmt):
    """cp_lse_combine_rank's contract, by the oracle: one destination."""
    def combine(recv_o, recv_lse, out=None, out_lse=None):
        ro = recv_o.view(torch.int16).numpy().view(np.uint16)
        W = ro.shape[0]
        _, ol, rounded = orc.combine(np.broadcast_to(ro, (W,) + ro.shape),
                                     np.broadcast_to(recv_lse.numpy(), (W,) + tuple(recv_lse.shape)),
                                     fmt)
        out.view(torch.int16).numpy()[...] = rounded[0].view(np.int16)
        out_lse.numpy()[...] = ol[0].astype(np.float32)
        return out, out_lse
    return combine


def _worker(rank, world, port, scatter_dim, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import synth
        from lse_pack_stable_b200.exchange import A2aExchange
        orc = oracle.get()
        wl = _workload(world)
        o, m, s = synth.full_inputs(wl)
        ex = A2aExchange(wl.T, wl.H, wl.D, torch.bfloat16, "cpu", scatter_dim=scatter_dim,
                         pack=_oracle_pack(orc), combine=_oracle_combine(orc, oracle.BF16))
        o_r = torch.from_numpy(o[rank].view(np.int16).copy()).view(torch.bfloat16)
        out_shape = ex.recv_o.shape[1:]
        out = torch.empty(out_shape, dtype=torch.bfloat16)
        out_lse = torch.empty(out_shape[:-1], dtype=torch.float32)
        ex(o_r, torch.from_numpy(m[rank].copy()), torch.from_numpy(s[rank].copy()), out, out_lse)
        q.put((rank, out.view(torch.int16).numpy().copy(), out_lse.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("scatter_dim", [1, 0])
def test_a2a_exchange_over_gloo(world, scatter_dim):
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    orc = oracle.get()
    wl = _workload(world)
    o, m, s = synth.full_inputs(wl)
    pk, l32, _ = orc.pack(o, m, s, scatter_dim)
    _, ref_lse, ref = orc.combine(orc.permute(pk, world), orc.permute(l32, world), oracle.BF16)

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, scatter_dim, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, ob, ol = q.get(timeout=120)
        got[r] = (ob, ol)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for j in range(world):
        ob, ol = got[j]
        assert np.array_equal(ob.view(np.uint16), ref[j]), "payload of destination %d" % j
        assert np.array_equal(ol.view(np.uint32), ref_lse[j].astype(np.float32).view(np.uint32))


def _uly_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        g = torch.Generator().manual_seed(99)
        B, S_l, H, D = 2, 5, 2 * world, 8
        x = torch.randint(-30000, 30000, (world, B, S_l, H, D), dtype=torch.int16, generator=g)
        y = bench.all_to_all_4d_nccl(x[rank].view(torch.bfloat16), 2, 1, world,
                                     (B, S_l * world, H // world, D))
        h = torch.randint(-30000, 30000, (world, B, S_l * world, H // world, D), dtype=torch.int16,
                          generator=g)
        z = bench.all_to_all_4d_nccl(h[rank].view(torch.bfloat16), 1, 2, world, (B, S_l, H, D))
        q.put((rank, y.view(torch.int16).numpy().copy(), z.view(torch.int16).numpy().copy(),
               x.numpy(), h.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_nccl_style_all_to_all_4d_reference(world):
    """The bench's NCCL-path reference for the Ulysses exchange (torch reshapes
    around all_to_all_single), run over gloo, equals the oracle's transforms."""
    sys.path.insert(0, ROOT)
    import oracle
    orc = oracle.get()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_uly_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, y, z, x, h = q.get(timeout=120)
        got[r] = (y, z)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    ref_y = orc.seq2head(x)
    ref_z = orc.head2seq(h)
    for r in range(world):
        assert np.array_equal(got[r][0], ref_y[r]), "seq->head rank %d" % r
        assert np.array_equal(got[r][1], ref_z[r]), "head->seq rank %d" % r
