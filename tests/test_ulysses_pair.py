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
    gen = torch.Generator(device="cuda").manual_seed(W * S_l + H)

    def bf16(shape, grad=False):
        return torch.randn(shape, device="cuda", dtype=torch.bfloat16, generator=gen,
                           requires_grad=grad)

    seq_shape, head_shape = (W, 3, S_l, H, D), (W, 3, S_l * W, H // W, D)
    qkv = bf16(seq_shape, grad=True)                                # sequence-sharded q/k/v
    attn = bf16((W, 1, S_l * W, H // W, D), grad=True)              # head-sharded attention output
    upstream_heads = bf16(head_shape)                               # d loss / d seq2head(qkv)
    upstream_seq = bf16((W, 1, S_l, H, D))                          # d loss / d head2seq(attn)
    heads = cp.ulysses_seq2head_autograd(qkv)
    tokens = cp.ulysses_head2seq_autograd(attn)
    grad_qkv, grad_attn = torch.autograd.grad(outputs=[heads, tokens], inputs=[qkv, attn],
                                              grad_outputs=[upstream_heads, upstream_seq])
    torch.cuda.synchronize()
    # forward: the layouts; backward: each gradient is the inverse layout of its upstream
    assert np.array_equal(_bits(heads), orc.seq2head(_bits(qkv)))
    assert np.array_equal(_bits(tokens), orc.head2seq(_bits(attn)))
    assert np.array_equal(_bits(grad_qkv), orc.head2seq(_bits(upstream_heads)))
    assert np.array_equal(_bits(grad_attn), orc.seq2head(_bits(upstream_seq)))


def test_pair_graph_capture_and_changed_input_replay():
    W, S_l, H, D = 8, 512, 48, 128
    qkv = torch.randn((W, 3, S_l, H, D), device="cuda", dtype=torch.bfloat16)
    attn = torch.randn((W, 1, S_l * W, H // W, D), device="cuda", dtype=torch.bfloat16)
    heads = torch.empty((W, 3, S_l * W, H // W, D), device="cuda", dtype=torch.bfloat16)
    tokens = torch.empty((W, 1, S_l, H, D), device="cuda", dtype=torch.bfloat16)

    def pair(stream=None):
        cp.ulysses_seq2head(qkv, out=heads, stream=stream)
        cp.ulysses_head2seq(attn, out=tokens, stream=stream)

    pair()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        pair(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    qkv.normal_()                       # new contents at the captured addresses
    attn.normal_()
    graph.replay()
    torch.cuda.synchronize()
    replayed = (heads.clone(), tokens.clone())
    pair()                              # eager on the same new inputs
    torch.cuda.synchronize()
    assert torch.equal(replayed[0].view(torch.int16), heads.view(torch.int16))
    assert torch.equal(replayed[1].view(torch.int16), tokens.view(torch.int16))
    assert torch.equal(cp.ulysses_head2seq(heads).view(torch.int16), qkv.view(torch.int16))
    del graph
