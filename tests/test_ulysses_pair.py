"""Ulysses training pair and graph replay.

The FastVideo page times a "training pair" (seq->head of q/k/v and head->seq
of the attention output, forward and backward through autograd, compared
bit-for-bit with the NCCL path) and a CUDA-graph capture of the pair replayed
after warm-up. Here: the autograd wrappers' gradients are the inverse layout
of the incoming gradients, bit-exact against the CPU oracle, and a captured
pair replayed on changed inputs matches eager execution.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

cp = pytest.importorskip("lse_pack_stable_b200")


def _bits(t):
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("W,S_l,H,D", [(2, 5, 4, 8), (4, 64, 8, 128), (8, 16, 48, 128)])
def test_training_pair_gradients(W, S_l, H, D, orc):
    g = torch.Generator(device="cuda").manual_seed(W * S_l + H)
    x = torch.randn((W, 3, S_l, H, D), device="cuda", dtype=torch.bfloat16, generator=g,
                    requires_grad=True)
    y = torch.randn((W, 1, S_l * W, H // W, D), device="cuda", dtype=torch.bfloat16, generator=g,
                    requires_grad=True)
    dx = torch.randn((W, 3, S_l * W, H // W, D), device="cuda", dtype=torch.bfloat16, generator=g)
    dy = torch.randn((W, 1, S_l, H, D), device="cuda", dtype=torch.bfloat16, generator=g)
    ox = cp.ulysses_seq2head_autograd(x)
    oy = cp.ulysses_head2seq_autograd(y)
    gx, gy = torch.autograd.grad((ox, oy), (x, y), (dx, dy))
    torch.cuda.synchronize()
    assert np.array_equal(_bits(ox), orc.seq2head(_bits(x)))
    assert np.array_equal(_bits(oy), orc.head2seq(_bits(y)))
    assert np.array_equal(_bits(gx), orc.head2seq(_bits(dx)))
    assert np.array_equal(_bits(gy), orc.seq2head(_bits(dy)))


def test_pair_graph_capture_and_changed_input_replay():
    W, S_l, H, D = 8, 512, 48, 128
    x = torch.randn((W, 3, S_l, H, D), device="cuda", dtype=torch.bfloat16)
    y = torch.randn((W, 1, S_l * W, H // W, D), device="cuda", dtype=torch.bfloat16)
    ox = torch.empty((W, 3, S_l * W, H // W, D), device="cuda", dtype=torch.bfloat16)
    oy = torch.empty((W, 1, S_l, H, D), device="cuda", dtype=torch.bfloat16)

    def pair(stream=None):
        cp.ulysses_seq2head(x, out=ox, stream=stream)
        cp.ulysses_head2seq(y, out=oy, stream=stream)

    pair()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        pair(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    x.normal_()
    y.normal_()
    graph.replay()
    torch.cuda.synchronize()
    got = (ox.clone(), oy.clone())
    pair()
    torch.cuda.synchronize()
    assert torch.equal(got[0].view(torch.int16), ox.view(torch.int16))
    assert torch.equal(got[1].view(torch.int16), oy.view(torch.int16))
    assert torch.equal(cp.ulysses_head2seq(ox).view(torch.int16), x.view(torch.int16))
    del graph
