"""CUDA-graph capture with changed-input replay.

The DCP pull request's test section ("How was this patch tested?") covers
CUDA-graph capture. The check here runs the call once without a graph,
captures it, and replays it. It then overwrites the inputs in place, at the
same addresses, and replays again: that replay has to produce the new results,
not the captured ones. The same sequence here, for the fused call and the
pack -> all-to-all -> combine chain, on a side stream.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import dev_f32, dev_payload

pytestmark = pytest.mark.gpu

cp = pytest.importorskip("lse_pack_stable_b200")


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def test_graph_capture_and_changed_input_replay():
    wl = synth.CONFIGS["decode"]
    W, T, H, D = wl.W, wl.T, wl.H, wl.D
    o, m, s = synth.full_inputs(wl)
    do, dm, ds = dev_payload(o, "bf16"), dev_f32(m), dev_f32(s)
    Hc = H // W
    out = torch.empty((W, T, Hc, D), dtype=torch.bfloat16, device="cuda")
    out_lse = torch.empty((W, T, Hc), dtype=torch.float32, device="cuda")
    pkt = torch.empty((W, W, T, Hc, D), dtype=torch.bfloat16, device="cuda")
    pl = torch.empty((W, W, T, Hc), dtype=torch.float32, device="cuda")
    ro, rl = torch.empty_like(pkt), torch.empty_like(pl)
    co, cl = torch.empty_like(out), torch.empty_like(out_lse)
    tout = torch.empty((W, T // W, H, D), dtype=torch.bfloat16, device="cuda")
    tlse = torch.empty((W, T // W, H), dtype=torch.float32, device="cuda")
    results = (out, out_lse, co, cl, tout, tlse)

    def step(stream=None):
        cp.cp_pack_permute_combine_fused(do, dm, ds, out=out, out_lse=out_lse, stream=stream)
        cp.cp_pack_permute_combine_fused(do, dm, ds, out=tout, out_lse=tlse, scatter_dim=0,
                                         stream=stream)
        cp.cp_pack_lse(do, dm, ds, pkt_o=pkt, pkt_lse=pl, stream=stream)
        cp.cp_a2a_local_permute(pkt, W, recv=ro, stream=stream)
        cp.cp_a2a_local_permute(pl, W, recv=rl, stream=stream)
        cp.cp_lse_combine(ro, rl, out=co, out_lse=cl, stream=stream)

    step()
    torch.cuda.synchronize()
    eager = [_bits(t).clone() for t in results]

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    for t in results:
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for want, got in zip(eager, results):
        assert torch.equal(want, _bits(got))

    # change the inputs in place (same addresses), replay, compare with eager
    wl2 = synth.Workload("decode2", W=W, T=T, H=H, D=D, seed=77, max_sigma=5.0,
                         sum_dist=(synth.UNIFORM, 1.0, 4096.0), p_invalid=0.02)
    o2, m2, s2 = synth.full_inputs(wl2)
    do.copy_(dev_payload(o2, "bf16"))
    dm.copy_(dev_f32(m2))
    ds.copy_(dev_f32(s2))
    graph.replay()
    torch.cuda.synchronize()
    replayed = [_bits(t).clone() for t in results]
    assert not torch.equal(replayed[0], eager[0]), "replay returned stale results"
    step()
    torch.cuda.synchronize()
    for want, got in zip(replayed, results):
        assert torch.equal(want, _bits(got))
    assert torch.equal(replayed[0], replayed[2]) and torch.equal(replayed[1], replayed[3])
    # token chunks: the head-chunk rows in source order
    assert torch.equal(replayed[0].transpose(0, 1).reshape(T, H, D), replayed[4].reshape(T, H, D))
    assert torch.equal(replayed[1].transpose(0, 1).reshape(T, H), replayed[5].reshape(T, H))
    del graph


def test_graph_exchange_entry_points_changed_input_replay():
    """The two-rank regression of the DCP page (eager, capture, first replay,
    changed-input replay at fixed addresses) for the entry points of the
    exchange across real ranks, W = 2 ranks held as separate planes on this
    GPU: each rank's pack, the all-to-all as block copies between the send and
    receive buffers, each destination's combine, and the pull kernel."""
    wl = synth.Workload("pair", W=2, T=512, H=16, D=128, dtype="bf16", seed=5, max_sigma=5.0,
                        sum_dist=(synth.UNIFORM, 1.0, 512.0), p_invalid=0.03)
    W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
    o, m, s = synth.full_inputs(wl)
    planes = [dev_payload(o[r], "bf16") for r in range(W)]
    mpl = [dev_f32(m[r]) for r in range(W)]
    spl = [dev_f32(s[r]) for r in range(W)]
    send = [(torch.empty((W, T, Hc, D), dtype=torch.bfloat16, device="cuda"),
             torch.empty((W, T, Hc), dtype=torch.float32, device="cuda")) for _ in range(W)]
    recv = [(torch.empty((W, T, Hc, D), dtype=torch.bfloat16, device="cuda"),
             torch.empty((W, T, Hc), dtype=torch.float32, device="cuda")) for _ in range(W)]
    outs = [(torch.empty((T, Hc, D), dtype=torch.bfloat16, device="cuda"),
             torch.empty((T, Hc), dtype=torch.float32, device="cuda")) for _ in range(2 * W)]

    def step(stream=None):
        for r in range(W):
            cp.cp_pack_lse_rank(planes[r], mpl[r], spl[r], W, pkt_o=send[r][0],
                                pkt_lse=send[r][1], stream=stream)
        # the all-to-all: block j of rank r's packet lands as block r at rank j
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            for j in range(W):
                for r in range(W):
                    recv[j][0][r].copy_(send[r][0][j])
                    recv[j][1][r].copy_(send[r][1][j])
        for j in range(W):
            cp.cp_lse_combine_rank(recv[j][0], recv[j][1], out=outs[j][0], out_lse=outs[j][1],
                                   stream=stream)
            cp.cp_pull_combine(planes, mpl, spl, j, out=outs[W + j][0], out_lse=outs[W + j][1],
                               stream=stream)

    results = [t for pair in outs for t in pair]
    step()
    torch.cuda.synchronize()
    eager = [_bits(t).clone() for t in results]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    for t in results:
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for want, got in zip(eager, results):
        assert torch.equal(want, _bits(got))

    wl2 = synth.Workload("pair2", W=W, T=T, H=H, D=D, seed=91, max_sigma=5.0,
                         sum_dist=(synth.UNIFORM, 1.0, 512.0), p_invalid=0.05)
    o2, m2, s2 = synth.full_inputs(wl2)
    for r in range(W):
        planes[r].copy_(dev_payload(o2[r], "bf16"))
        mpl[r].copy_(dev_f32(m2[r]))
        spl[r].copy_(dev_f32(s2[r]))
    graph.replay()
    torch.cuda.synchronize()
    replayed = [_bits(t).clone() for t in results]
    assert not torch.equal(replayed[0], eager[0]), "replay returned stale results"
    fo, fl = cp.cp_pack_permute_combine_fused(torch.stack(planes), torch.stack(mpl),
                                              torch.stack(spl))
    torch.cuda.synchronize()
    for j in range(W):      # both paths give destination j of the fused call
        for k in (j, W + j):
            assert torch.equal(replayed[2 * k], _bits(fo[j]))
            assert torch.equal(replayed[2 * k + 1], _bits(fl[j]))
    del graph
