"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times.

Inputs are generated on the host block by block and uploaded. The oracle
checks sampled output rows one by one: for each sampled (t, h) the generator
regenerates that row's W partial outputs and statistics, and the oracle merges
them (``fused_gathered``). Properties that hold at any size are checked over
every element on the device: the unfused pack -> all-to-all -> combine chain
equals the fused kernel bit for bit, and so do the entry points of the
exchange across GPUs (the pull kernel for every destination, one rank's pack,
one destination's combine), run here on the W planes of one GPU. The Ulysses
transforms are compared with the oracle in full, and their pull form with
them.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import (FMT, TORCH_DT, check_combined, check_pack_lse, host_bits,
                      lse_member_tol)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

cp = pytest.importorskip("lse_pack_stable_b200")

CONFIG_NAMES = ["decode", "mla", "ulysses", "stress"]


def device_inputs(wl: synth.Workload):
    """o [W,T,H,D], smax/ssum [W,T,H] on the device, uploaded in ~256 MB blocks."""
    W, T, H, D = wl.W, wl.T, wl.H, wl.D
    o = torch.empty((W, T, H, D), dtype=TORCH_DT[wl.dtype], device="cuda")
    m = torch.empty((W, T, H), dtype=torch.float32, device="cuda")
    s = torch.empty((W, T, H), dtype=torch.float32, device="cuda")
    tb = max(1, (256 << 20) // (H * D * 2))
    for r in range(W):
        for t0 in range(0, T, tb):
            t1 = min(T, t0 + tb)
            bits = synth.o_block(wl, r, t0, t1)
            o[r, t0:t1].view(torch.int16).copy_(torch.from_numpy(bits.view(np.int16)))
        mr, sr = synth.stats_block(wl, r)
        m[r].copy_(torch.from_numpy(mr))
        s[r].copy_(torch.from_numpy(sr))
    return o, m, s


def sample_rows(wl: synth.Workload, n: int = 1536, seed: int = 0):
    rng = np.random.default_rng(seed + wl.seed)
    t = rng.integers(0, wl.T, n)
    h = rng.integers(0, wl.H, n)
    edge_t = [0, 0, wl.T - 1, wl.T - 1, wl.T // 2]
    edge_h = [0, wl.H - 1, 0, wl.H - 1, wl.Hc]
    if wl.p_token_invalid > 0:   # a few whole invalid tokens
        bad = np.flatnonzero(synth.fill(wl.seed, synth.TID_BADTOK, synth.UNIT, 0, 0, n=wl.T,
                                        fmt=synth.F64) < wl.p_token_invalid)[:4]
        edge_t += bad.tolist()
        edge_h += [int(x) % wl.H for x in bad]
    return np.concatenate([t, edge_t]).astype(np.int64), np.concatenate([h, edge_h]).astype(np.int64)


def oracle_rows(wl, t, h, orc):
    o = np.stack([synth.o_rows(wl, r, t, h) for r in range(wl.W)])
    ms = [synth.stats_at(wl, r, t, h) for r in range(wl.W)]
    m = np.stack([a for a, _ in ms])
    s = np.stack([b for _, b in ms])
    ref, ref_lse, ref_r = orc.fused_gathered(o, m, s, FMT[wl.dtype])
    return o, m, s, ref, ref_lse, ref_r


@pytest.mark.parametrize("name", CONFIG_NAMES)
def test_fullsize_fused_and_chain(name, orc):
    wl = synth.CONFIGS[name]
    W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
    o, m, s = device_inputs(wl)
    out, out_lse = cp.cp_pack_permute_combine_fused(o, m, s)
    torch.cuda.synchronize()

    t, h = sample_rows(wl)
    j, hc = h // Hc, h % Hc
    ti, ji, hci = (torch.from_numpy(x).cuda() for x in (t, j, hc))
    got = host_bits(out[ji, ti, hci])
    got_lse = out_lse[ji, ti, hci].cpu().numpy()
    ro, rm, rs, ref, ref_lse, ref_r = oracle_rows(wl, t, h, orc)
    check_combined(got, got_lse, ref, ref_lse, ref_r, wl.dtype, W,
                   extra_lse_tol=lse_member_tol(rm, rs))

    # the pull kernel of the exchange across GPUs, every destination, reading the
    # W planes of this GPU's input: destination j of the fused result, bit for bit
    planes = ([o[r] for r in range(W)], [m[r] for r in range(W)], [s[r] for r in range(W)])
    for jj in range(W):
        po, pl_ = cp.cp_pull_combine(*planes, jj)
        torch.cuda.synchronize()
        assert torch.equal(po.view(torch.int16), out[jj].view(torch.int16)), "pull, dst %d" % jj
        assert torch.equal(pl_.view(torch.int32), out_lse[jj].view(torch.int32))
        del po, pl_

    # unfused chain on the full problem, then back to the sampled rows
    pkt, pl = cp.cp_pack_lse(o, m, s, scatter_dim=1)
    torch.cuda.synchronize()
    for r in (0, W - 1):          # one real rank's pack: plane r of the packet
        po, plr = cp.cp_pack_lse_rank(o[r], m[r], s[r], W)
        torch.cuda.synchronize()
        assert torch.equal(po.view(torch.int16), pkt[r].view(torch.int16)), "rank pack %d" % r
        assert torch.equal(plr.view(torch.int32), pl[r].view(torch.int32))
        del po, plr
    ri = torch.arange(W, device="cuda")[:, None]
    pk_rows = pkt[ri, ji[None], ti[None], hci[None]]          # [W, n, D]
    assert np.array_equal(host_bits(pk_rows), ro), "packet payload differs from the inputs"
    lse64 = np.vectorize(orc.lse)(rm.astype(np.float64), rs.astype(np.float64))
    check_pack_lse(pl[ri, ji[None], ti[None], hci[None]].cpu().numpy(), lse64, rm, rs)
    del o
    recv = cp.cp_a2a_local_permute(pkt, W)
    recv_l = cp.cp_a2a_local_permute(pl, W)
    del pkt
    torch.cuda.synchronize()
    rv_rows = recv[ji[None], ri, ti[None], hci[None]]          # recv[j][r][t][hc]
    assert np.array_equal(host_bits(rv_rows), ro), "received blocks differ from the inputs"
    co, cl = cp.cp_lse_combine(recv, recv_l)
    torch.cuda.synchronize()
    assert torch.equal(co.view(torch.int16), out.view(torch.int16)), "chain != fused"
    assert torch.equal(cl.view(torch.int32), out_lse.view(torch.int32)), "chain LSE != fused"
    for jj in (0, W - 1):         # one real destination's combine
        oj, lj = cp.cp_lse_combine_rank(recv[jj], recv_l[jj])
        torch.cuda.synchronize()
        assert torch.equal(oj.view(torch.int16), out[jj].view(torch.int16)), "rank combine %d" % jj
        assert torch.equal(lj.view(torch.int32), out_lse[jj].view(torch.int32))
        del oj, lj
    del recv, recv_l, co, cl, out, out_lse, m, s
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", CONFIG_NAMES)
def test_fullsize_token_scatter(name, orc):
    """The token-chunk exchange at full size: sampled rows against the oracle,
    and every element against the head-chunk result it permutes."""
    wl = synth.CONFIGS[name]
    W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
    Tc = T // W
    o, m, s = device_inputs(wl)
    tok, tok_lse = cp.cp_pack_permute_combine_fused(o, m, s, scatter_dim=0)
    torch.cuda.synchronize()
    t, h = sample_rows(wl, seed=1)
    ti, hi = (torch.from_numpy(x).cuda() for x in (t, h))
    got = host_bits(tok[ti // Tc, ti % Tc, hi])
    got_lse = tok_lse[ti // Tc, ti % Tc, hi].cpu().numpy()
    _, rm, rs, ref, ref_lse, ref_r = oracle_rows(wl, t, h, orc)
    check_combined(got, got_lse, ref, ref_lse, ref_r, wl.dtype, W,
                   extra_lse_tol=lse_member_tol(rm, rs))
    head, head_lse = cp.cp_pack_permute_combine_fused(o, m, s, scatter_dim=1)
    torch.cuda.synchronize()
    del o, m, s
    assert torch.equal(head.view(torch.int16).transpose(0, 1).reshape(T, H, D),
                       tok.view(torch.int16).reshape(T, H, D)), "token != permuted head result"
    assert torch.equal(head_lse.view(torch.int32).transpose(0, 1).reshape(T, H),
                       tok_lse.view(torch.int32).reshape(T, H))
    del head, head_lse, tok, tok_lse
    torch.cuda.empty_cache()


def test_fullsize_ulysses(orc):
    wl = synth.CONFIGS["ulysses"]
    W, S_l = wl.W, wl.T // wl.W
    xs = np.stack([synth.ulysses_seq_block(wl, r) for r in range(W)])       # [W,3,S_l,H,D]
    xd = torch.from_numpy(xs.view(np.int16)).cuda().view(torch.bfloat16)
    y = cp.ulysses_seq2head(xd)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(y), orc.seq2head(xs))
    back = cp.ulysses_head2seq(y)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), xd.view(torch.int16))
    # the load/store exchange across GPUs, every destination, from this GPU's planes
    for j in range(W):
        yj = cp.ulysses_seq2head_pull([xd[r] for r in range(W)], j)
        bj = cp.ulysses_head2seq_pull([y[r] for r in range(W)], j)
        torch.cuda.synchronize()
        assert torch.equal(yj.view(torch.int16), y[j].view(torch.int16)), "seq2head pull %d" % j
        assert torch.equal(bj.view(torch.int16), xd[j].view(torch.int16)), "head2seq pull %d" % j
        del yj, bj
    del xd, y, back
    xh = np.stack([synth.ulysses_head_block(wl, r) for r in range(W)])      # [W,1,S,Hc,D]
    hd = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
    z = cp.ulysses_head2seq(hd)
    torch.cuda.synchronize()
    assert z.shape == (W, 1, S_l, wl.H, wl.D)
    assert np.array_equal(host_bits(z), orc.head2seq(xh))
