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
