"""The entry points of the exchange across real ranks, on one GPU.

* cp_pack_lse_rank on plane r equals plane r of cp_pack_lse's W-rank packet,
  and the oracle's, bit for bit;
* cp_lse_combine_rank on destination j's received packet equals destination j
  of cp_lse_combine, bit for bit, and meets the combine tolerances against
  the oracle;
* cp_pull_combine for destination j, reading W separately allocated planes
  through its pointer table (contiguous and strided), equals destination j of
  cp_pack_permute_combine_fused bit for bit, in both scatter modes;
* PullExchange end to end with 2 and 3 processes sharing this GPU: each maps
  the others' planes through CUDA IPC and pulls its destination; the results
  equal the fused call's blocks. The processes synchronise on the host (gloo);
  no kernel waits for another.
"""
from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch

import synth
from gpu_util import FMT, check_combined, check_pack_lse, dev_f32, dev_payload, host_bits
from test_parity import CASES, IDS, TOKEN_CASES, _packet_layout, _scatter_params, _wl

pytestmark = pytest.mark.gpu

cp = pytest.importorskip("lse_pack_stable_b200")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _dev(wl):
    o, m, s = synth.full_inputs(wl)
    return (o, m, s), (dev_payload(o, wl.dtype), dev_f32(m), dev_f32(s))


@pytest.mark.parametrize("wl,scatter_dim", _scatter_params(CASES))
def test_pack_rank_is_a_plane_of_the_pack(wl, scatter_dim, orc):
    (o, m, s), (do, dm, ds) = _dev(wl)
    pkt, pl = cp.cp_pack_lse(do, dm, ds, scatter_dim=scatter_dim)
    ref_o, _, ref_l = orc.pack(o, m, s, scatter_dim)
    W, T, H = wl.W, wl.T, wl.H
    for r in range(W):
        po, plr = cp.cp_pack_lse_rank(do[r], dm[r], ds[r], W, scatter_dim=scatter_dim)
        torch.cuda.synchronize()
        assert torch.equal(po.view(torch.int16), pkt[r].view(torch.int16)), "payload, plane %d" % r
        assert torch.equal(plr.view(torch.int32), pl[r].view(torch.int32)), "LSE, plane %d" % r
        assert np.array_equal(host_bits(po), ref_o[r])
    check_pack_lse(pl.cpu().numpy(), ref_l, _packet_layout(m, W, T, H, scatter_dim),
                   _packet_layout(s, W, T, H, scatter_dim))


def test_pack_rank_strided_plane():
    wl = _wl("rank_strided", 4, 13, 8, 64, p_invalid=0.1)
    (o, m, s), (do, dm, ds) = _dev(wl)
    big = torch.zeros((wl.T + 2, wl.H + 3, wl.D + 8), dtype=torch.bfloat16, device="cuda")
    ov = big[1:wl.T + 1, 2:wl.H + 2, 8:]
    bm = torch.zeros((wl.T, 2 * wl.H), dtype=torch.float32, device="cuda")
    pkt, pl = cp.cp_pack_lse(do, dm, ds)
    for r in range(wl.W):
        ov.copy_(do[r])
        mv = bm[:, 1::2]
        mv.copy_(dm[r])
        sv = ds[r].t().contiguous().t()
        po, plr = cp.cp_pack_lse_rank(ov, mv, sv, wl.W)
        torch.cuda.synchronize()
        assert torch.equal(po.view(torch.int16), pkt[r].view(torch.int16))
        assert torch.equal(plr.view(torch.int32), pl[r].view(torch.int32))


@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_combine_rank_is_a_destination_of_the_combine(wl, orc):
    (o, m, s), (do, dm, ds) = _dev(wl)
    pkt, pl = cp.cp_pack_lse(do, dm, ds)
    ro, rl = cp.cp_a2a_local_permute(pkt, wl.W), cp.cp_a2a_local_permute(pl, wl.W)
    out, out_lse = cp.cp_lse_combine(ro, rl)
    ref_pkt, l32, _ = orc.pack(o, m, s, 1)
    ref, ref_lse, ref_r = orc.combine(orc.permute(ref_pkt, wl.W), orc.permute(l32, wl.W),
                                      FMT[wl.dtype])
    for j in range(wl.W):
        oj, lj = cp.cp_lse_combine_rank(ro[j], rl[j])
        torch.cuda.synchronize()
        assert torch.equal(oj.view(torch.int16), out[j].view(torch.int16)), "destination %d" % j
        assert torch.equal(lj.view(torch.int32), out_lse[j].view(torch.int32))
        check_combined(host_bits(oj), lj.cpu().numpy(), ref[j], ref_lse[j], ref_r[j], wl.dtype,
                       wl.W)


@pytest.mark.parametrize("wl", [w for w in TOKEN_CASES if w.T % w.W == 0][:6],
                         ids=[w.name for w in TOKEN_CASES if w.T % w.W == 0][:6])
def test_combine_rank_on_token_chunks(wl):
    """The token-chunk packet: destination j's received [W, T/W, H, D] is
    combined with T/W as T and H as Hc, and equals destination j of the
    W-rank combine and of the token-chunk fused call."""
    (o, m, s), (do, dm, ds) = _dev(wl)
    pkt, pl = cp.cp_pack_lse(do, dm, ds, scatter_dim=0)
    ro, rl = cp.cp_a2a_local_permute(pkt, wl.W), cp.cp_a2a_local_permute(pl, wl.W)
    out, out_lse = cp.cp_lse_combine(ro, rl)
    fo, fl = cp.cp_pack_permute_combine_fused(do, dm, ds, scatter_dim=0)
    for j in range(wl.W):
        oj, lj = cp.cp_lse_combine_rank(ro[j], rl[j])
        torch.cuda.synchronize()
        assert torch.equal(oj.view(torch.int16), out[j].view(torch.int16)), "destination %d" % j
        assert torch.equal(lj.view(torch.int32), out_lse[j].view(torch.int32))
        assert torch.equal(oj.view(torch.int16), fo[j].view(torch.int16))
        assert torch.equal(lj.view(torch.int32), fl[j].view(torch.int32))


def _separate_planes(do, dm, ds, strided):
    """W separately allocated planes per tensor (optionally strided views)."""
    os_, ms, ss = [], [], []
    for r in range(do.shape[0]):
        if strided:
            T, H, D = do.shape[1:]
            big = torch.zeros((T, H + 1, D + 8), dtype=do.dtype, device="cuda")
            v = big[:, 1:, 8:]
            v.copy_(do[r])
            os_.append(v)
            bm = torch.zeros((T, 3 * H), dtype=torch.float32, device="cuda")
            mv = bm[:, ::3]
            mv.copy_(dm[r])
            ms.append(mv)
            bs = torch.zeros((T, 2 * H), dtype=torch.float32, device="cuda")
            sv = bs[:, 1::2]
            sv.copy_(ds[r])
            ss.append(sv)
        else:
            os_.append(do[r].clone())
            ms.append(dm[r].clone())
            ss.append(ds[r].clone())
    return os_, ms, ss


@pytest.mark.parametrize("wl,scatter_dim", _scatter_params(CASES, TOKEN_CASES))
def test_pull_equals_fused_destination(wl, scatter_dim):
    (o, m, s), (do, dm, ds) = _dev(wl)
    fo, fl = cp.cp_pack_permute_combine_fused(do, dm, ds, scatter_dim=scatter_dim)
    planes = _separate_planes(do, dm, ds, strided=False)
    for j in range(wl.W):
        oj, lj = cp.cp_pull_combine(*planes, j, scatter_dim=scatter_dim)
        torch.cuda.synchronize()
        assert torch.equal(oj.view(torch.int16), fo[j].view(torch.int16)), "destination %d" % j
        assert torch.equal(lj.view(torch.int32), fl[j].view(torch.int32))


@pytest.mark.parametrize("wl", [CASES[1], CASES[3], CASES[8], CASES[9]],
                         ids=[IDS[1], IDS[3], IDS[8], IDS[9]])
def test_pull_strided_planes_against_the_oracle(wl, orc):
    (o, m, s), (do, dm, ds) = _dev(wl)
    planes = _separate_planes(do, dm, ds, strided=True)
    ref, ref_lse, ref_r = orc.fused(o, m, s, FMT[wl.dtype])
    fo, fl = cp.cp_pack_permute_combine_fused(do, dm, ds)
    for j in range(wl.W):
        oj, lj = cp.cp_pull_combine(*planes, j)
        torch.cuda.synchronize()
        assert torch.equal(oj.view(torch.int16), fo[j].view(torch.int16))
        # tolerances against the float64 oracle (the LSE of each contribution is
        # formed on the fly, as in the fused path: its bound adds in)
        from gpu_util import lse_member_tol
        W, T, H = wl.W, wl.T, wl.H
        tol = lse_member_tol(m.reshape(W, -1), s.reshape(W, -1)).reshape(T, W, H // W)[:, j]
        check_combined(host_bits(oj), lj.cpu().numpy(), ref[j], ref_lse[j], ref_r[j], wl.dtype,
                       W, extra_lse_tol=tol)


def test_pull_rejects_misshapen_planes():
    wl = CASES[0]
    (o, m, s), (do, dm, ds) = _dev(wl)
    planes = list(_separate_planes(do, dm, ds, strided=False))
    with pytest.raises(ValueError):
        cp.cp_pull_combine(planes[0], planes[1][:1], planes[2], 0)
    with pytest.raises(cp.CplseError, match="dst"):
        cp.cp_pull_combine(*planes, wl.W)
    host = [p.cpu() for p in planes[0]]
    with pytest.raises(cp.CplseError, match="not device memory"):
        cp.cp_pull_combine(host, planes[1], planes[2], 0)


# --------------------------------------------------------------------- processes sharing one GPU

def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _pull_worker(rank, world, port, wl, scatter_dim, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ex = None
    try:
        import synth as sy
        from gpu_util import dev_f32 as f32, dev_payload as pay
        from lse_pack_stable_b200.exchange import PullExchange
        o, m, s = sy.full_inputs(wl)
        ex = PullExchange(wl.T, wl.H, wl.D, pay(o[:1], wl.dtype).dtype, "cuda:0",
                          scatter_dim=scatter_dim)
        res = []
        side = torch.cuda.Stream()
        for step in range(2):             # the second step overwrites the planes
            scale = 1 if step == 0 else -1
            ex.o.copy_(pay(o[rank], wl.dtype) * scale)
            ex.smax.copy_(f32(m[rank]))
            ex.ssum.copy_(f32(s[rank]))
            if step == 0:
                out, out_lse = ex()
            else:                         # on a side stream: the barriers order that stream
                side.wait_stream(torch.cuda.current_stream())
                out, out_lse = ex(stream=side)
            torch.cuda.synchronize()
            res.append((out.view(torch.int16).cpu().numpy(), out_lse.cpu().numpy()))
        q.put((rank, res))
    except Exception as e:  # noqa: BLE001
        q.put((rank, repr(e)))
        raise
    finally:
        if ex is not None:
            ex.close()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,scatter_dim", [(2, 1), (3, 1), (2, 0)])
def test_pull_exchange_processes_on_one_gpu(world, scatter_dim):
    import torch.multiprocessing as mp
    wl = _wl("ipc_w%d" % world, world, 12 * world, 4 * world, 64, p_invalid=0.1)
    o, m, s = synth.full_inputs(wl)
    do, dm, ds = dev_payload(o, wl.dtype), dev_f32(m), dev_f32(s)
    refs = [cp.cp_pack_permute_combine_fused(do * sc, dm, ds, scatter_dim=scatter_dim)
            for sc in (1, -1)]
    torch.cuda.synchronize()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_pull_worker, args=(r, world, port, wl, scatter_dim, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, res = q.get(timeout=240)
        got[r] = res
    for p in procs:
        p.join(120)
    for r in range(world):
        assert not isinstance(got[r], str), got[r]
        for step, (out, out_lse) in enumerate(got[r]):
            fo, fl = refs[step]
            assert np.array_equal(out, fo[r].view(torch.int16).cpu().numpy()), (r, step)
            assert np.array_equal(out_lse.view(np.uint32),
                                  fl[r].cpu().numpy().view(np.uint32)), (r, step)
    assert all(p.exitcode == 0 for p in procs)


# --------------------------------------------------------------------- Ulysses across real ranks

@pytest.mark.parametrize("W,B,S_l,H,D,dtype", [(2, 1, 8, 4, 64, torch.bfloat16),
                                                (4, 3, 16, 8, 128, torch.bfloat16),
                                                (3, 2, 5, 6, 24, torch.float16),
                                                (8, 1, 64, 48, 128, torch.bfloat16),
                                                (4, 2, 7, 4, 3, torch.uint8),
                                                (2, 2, 9, 2, 5, torch.float32),
                                                (5, 1, 4, 10, 6, torch.float64)])
def test_ulysses_pull_equals_the_emulation(W, B, S_l, H, D, dtype, orc):
    g = torch.Generator().manual_seed(W * 100 + D)
    x = torch.randint(0, 255, (W, B, S_l, H, D * torch.empty((), dtype=dtype).element_size()),
                      dtype=torch.uint8, generator=g).view(dtype).cuda()
    y = cp.ulysses_seq2head(x)
    ranks = [x[r].clone() for r in range(W)]
    for j in range(W):
        yj = cp.ulysses_seq2head_pull(ranks, j)
        torch.cuda.synchronize()
        assert torch.equal(yj.view(torch.uint8), y[j].view(torch.uint8)), "seq2head dst %d" % j
    heads = [y[r].clone() for r in range(W)]
    for j in range(W):
        xj = cp.ulysses_head2seq_pull(heads, j)
        torch.cuda.synchronize()
        assert torch.equal(xj.view(torch.uint8), x[j].view(torch.uint8)), "head2seq dst %d" % j
    if dtype == torch.bfloat16:
        ref = orc.seq2head(x.view(torch.int16).cpu().numpy())
        assert np.array_equal(y.view(torch.int16).cpu().numpy(), ref)


def _uly_worker(rank, world, port, shape, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ex = None
    try:
        from lse_pack_stable_b200.exchange import UlyssesPullExchange
        B, S_l, H, D = shape
        g = torch.Generator().manual_seed(1234)
        x = torch.randn((world, B, S_l, H, D), generator=g).to(torch.bfloat16).cuda()
        ex = UlyssesPullExchange(B, B, S_l * world, H, D, torch.bfloat16, "cuda:0")
        ex.seq.copy_(x[rank])
        y = ex.seq2head()
        ex.head.copy_(y)                      # the head shard that comes back
        back = ex.head2seq()
        torch.cuda.synchronize()
        q.put((rank, y.view(torch.int16).cpu().numpy(), back.view(torch.int16).cpu().numpy()))
    except Exception as e:  # noqa: BLE001
        q.put((rank, repr(e), None))
        raise
    finally:
        if ex is not None:
            ex.close()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ulysses_pull_exchange_processes_on_one_gpu(world):
    import torch.multiprocessing as mp
    shape = (2, 6, 2 * world, 64)
    g = torch.Generator().manual_seed(1234)
    x = torch.randn((world,) + shape, generator=g).to(torch.bfloat16).cuda()
    y = cp.ulysses_seq2head(x)
    torch.cuda.synchronize()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_uly_worker, args=(r, world, port, shape, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, yr, back = q.get(timeout=240)
        got[r] = (yr, back)
    for p in procs:
        p.join(120)
    for r in range(world):
        yr, back = got[r]
        assert not isinstance(yr, str), yr
        assert np.array_equal(yr, y[r].view(torch.int16).cpu().numpy()), "seq2head rank %d" % r
        assert np.array_equal(back, x[r].view(torch.int16).cpu().numpy()), "round trip rank %d" % r
    assert all(p.exitcode == 0 for p in procs)
