"""The Python binding refuses tensors whose shape, dtype or device disagree with
the sizes it passes to the C layer (which derives every extent from W, T, H, D
and would otherwise read or write out of bounds). These checks run before any
pointer reaches the library, so they need no GPU: CPU tensors stand in."""
from __future__ import annotations

import pytest
import torch

import lse_pack_stable_b200 as cp

W, T, H, D = 2, 4, 8, 16
BF = torch.bfloat16


def _inputs():
    return (torch.zeros((W, T, H, D), dtype=BF), torch.zeros((W, T, H)), torch.zeros((W, T, H)))


def test_pack_rejects_undersized_packet():
    o, m, s = _inputs()
    with pytest.raises(ValueError, match="pkt_o"):
        cp.cp_pack_lse(o, m, s, pkt_o=torch.empty((W, W, T, H // W - 1, D), dtype=BF))
    with pytest.raises(ValueError, match="pkt_lse"):
        cp.cp_pack_lse(o, m, s, pkt_o=torch.empty((W, W, T, H // W, D), dtype=BF),
                       pkt_lse=torch.empty((W, W, T, H // W), dtype=torch.float64))


def test_pack_rejects_bad_statistics():
    o, m, s = _inputs()
    with pytest.raises(ValueError, match="smax"):
        cp.cp_pack_lse(o, m[:, :-1], s)
    with pytest.raises(ValueError, match="ssum"):
        cp.cp_pack_lse(o, m, s.double())
    with pytest.raises(ValueError, match="not a multiple"):
        cp.cp_pack_lse(o[:, :3], m[:, :3], s[:, :3], scatter_dim=0)


def test_fused_rejects_wrong_outputs():
    o, m, s = _inputs()
    with pytest.raises(ValueError, match="out"):
        cp.cp_pack_permute_combine_fused(o, m, s, out=torch.empty((W, T, H // W, D - 8), dtype=BF))
    with pytest.raises(ValueError, match="out"):
        cp.cp_pack_permute_combine_fused(o, m, s, out=torch.empty((W, T, H // W, D),
                                                                  dtype=torch.float16))
    with pytest.raises(ValueError, match="out_lse"):
        cp.cp_pack_permute_combine_fused(o, m, s, out_lse=torch.empty((W, T, H)))
    with pytest.raises(TypeError):
        cp.cp_pack_permute_combine_fused(o.float(), m, s)


def test_combine_rejects_mismatched_packet():
    ro = torch.zeros((W, W + 1, T, H // W, D), dtype=BF)
    rl = torch.zeros((W, W + 1, T, H // W))
    with pytest.raises(ValueError, match=r"\[W, W, T, Hc, D\]"):
        cp.cp_lse_combine(ro, rl)
    ro = torch.zeros((W, W, T, H // W, D), dtype=BF)
    with pytest.raises(ValueError, match="recv_lse"):
        cp.cp_lse_combine(ro, torch.zeros((W, W, T, H // W - 1)))
    with pytest.raises(ValueError, match="out"):
        cp.cp_lse_combine(ro, torch.zeros((W, W, T, H // W)),
                          out=torch.empty((W, T - 1, H // W, D), dtype=BF))


def test_materialize_and_pack_from_lse_shapes():
    o, m, s = _inputs()
    with pytest.raises(ValueError, match="lse"):
        cp.cp_lse_materialize(m, s, lse=torch.empty((W, T, H - 1)))
    with pytest.raises(ValueError, match="lse"):
        cp.cp_pack_from_lse(o, torch.zeros((W, T, H + 1)))


def test_permute_rejects_short_receive_buffer():
    send = torch.zeros(W * W * 64, dtype=torch.uint8)
    with pytest.raises(ValueError, match="recv"):
        cp.cp_a2a_local_permute(send, W, recv=torch.empty(W * W * 64 - 16, dtype=torch.uint8))


def test_ulysses_shapes():
    x = torch.zeros((W, 1, 3, H, D), dtype=BF)
    with pytest.raises(ValueError, match="out"):
        cp.ulysses_seq2head(x, out=torch.empty((W, 1, 3 * W, H // W, D - 1), dtype=BF))
    with pytest.raises(ValueError, match="not a multiple"):
        cp.ulysses_head2seq(torch.zeros((W, 1, 5, H // W, D), dtype=BF))
    with pytest.raises(ValueError, match="out"):
        cp.ulysses_head2seq(torch.zeros((W, 1, 6, H // W, D), dtype=BF),
                            out=torch.empty((W, 1, 3, H, D), dtype=torch.float16))

