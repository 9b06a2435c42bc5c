"""Bit-level identities of the GPU path that hold at any size.

- fused == pack -> all-to-all (both regions) -> combine, bit for bit: the fused
  kernel only moves where each LSE is formed, not how;
- W = 1 is the identity: O = O_0 and LSE* = LSE_0 exactly (exp(0) = 1, log 1 = 0);
- a row with a single valid contribution returns that contribution exactly;
- all-invalid rows give +0 and -inf;
- Ulysses head->seq undoes seq->head.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import dev_f32, dev_payload, host_bits

pytestmark = pytest.mark.gpu

cp = pytest.importorskip("lse_pack_stable_b200")


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def _chain(o, m, s, W):
    pkt, pl = cp.cp_pack_lse(o, m, s, scatter_dim=1)
    ro = cp.cp_a2a_local_permute(pkt, W)
    rl = cp.cp_a2a_local_permute(pl, W)
    return cp.cp_lse_combine(ro, rl)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_fused_equals_chain_configs(name):
    wl = synth.CONFIGS[name]
    o, m, s = synth.full_inputs(wl)
    do, dm, ds = dev_payload(o, wl.dtype), dev_f32(m), dev_f32(s)
    fo, fl = cp.cp_pack_permute_combine_fused(do, dm, ds)
    co, cl = _chain(do, dm, ds, wl.W)
    torch.cuda.synchronize()
    assert torch.equal(_bits(fo), _bits(co))
    assert torch.equal(_bits(fl), _bits(cl))


@pytest.mark.parametrize("W,T,H,D,dtype", [(3, 29, 9, 40, "fp16"), (16, 8, 32, 128, "fp16"),
                                           (32, 3, 32, 512, "bf16"), (8, 70, 16, 1024, "bf16")])
def test_fused_equals_chain_shapes(W, T, H, D, dtype):
    wl = synth.Workload("x", W=W, T=T, H=H, D=D, dtype=dtype, seed=W * T, max_sigma=9.0,
                        sum_dist=(synth.LOGUNIFORM, 1e-3, 1e6), p_invalid=0.05,
                        p_max_inf=0.02, p_sum_zero=0.02)
    o, m, s = synth.full_inputs(wl)
    do, dm, ds = dev_payload(o, dtype), dev_f32(m), dev_f32(s)
    fo, fl = cp.cp_pack_permute_combine_fused(do, dm, ds)
    co, cl = _chain(do, dm, ds, W)
    torch.cuda.synchronize()
    assert torch.equal(_bits(fo), _bits(co))
    assert torch.equal(_bits(fl), _bits(cl))


@pytest.mark.parametrize("W,T,H,D,dtype", [(4, 4096, 32, 128, "bf16"), (3, 33, 9, 40, "fp16"),
                                           (16, 32, 32, 128, "fp16"), (8, 16, 16, 512, "bf16")])
def test_token_scatter_is_a_permutation_of_head_scatter(W, T, H, D, dtype):
    """Both exchanges merge the same W contributions of each (t, h) in the same
    order; only where the row lands differs. Head chunks put (t, j*Hc + hc) at
    [j][t][hc], token chunks put (t, h) at [t // Tc][t % Tc][h]."""
    wl = synth.Workload("perm", W=W, T=T, H=H, D=D, dtype=dtype, seed=T + D, p_invalid=0.05,
                        max_sigma=9.0, sum_dist=(synth.LOGUNIFORM, 1e-3, 1e6))
    o, m, s = synth.full_inputs(wl)
    do, dm, ds = dev_payload(o, dtype), dev_f32(m), dev_f32(s)
    ho, hl = cp.cp_pack_permute_combine_fused(do, dm, ds, scatter_dim=1)
    to, tl = cp.cp_pack_permute_combine_fused(do, dm, ds, scatter_dim=0)
    torch.cuda.synchronize()
    assert torch.equal(_bits(ho).transpose(0, 1).reshape(T, H, D), _bits(to).reshape(T, H, D))
    assert torch.equal(_bits(hl).transpose(0, 1).reshape(T, H), _bits(tl).reshape(T, H))


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_w1_identity(dtype):
    wl = synth.Workload("w1", W=1, T=300, H=5, D=136, dtype=dtype, seed=3, p_invalid=0.0,
                        max_sigma=20.0, sum_dist=(synth.LOGUNIFORM, 1e-30, 1e30))
    o, m, s = synth.full_inputs(wl)
    o = o.copy()
    o.reshape(-1)[::7] = 0x8000          # -0.0 must survive too
    do, dm, ds = dev_payload(o, dtype), dev_f32(m), dev_f32(s)
    fo, fl = cp.cp_pack_permute_combine_fused(do, dm, ds)
    pkt, pl = cp.cp_pack_lse(do, dm, ds)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(fo), o)
    assert torch.equal(_bits(fl).reshape(-1), _bits(pl).reshape(-1))


def test_single_valid_contribution_is_exact():
    W, T, H, D = 8, 40, 16, 128
    wl = synth.Workload("one", W=W, T=T, H=H, D=D, seed=5, p_invalid=0.0)
    o, m, s = synth.full_inputs(wl)
    s = s.copy()
    keep = np.arange(T * H).reshape(T, H) % W            # the one valid rank of each (t, h)
    for r in range(W):
        s[r][keep != r] = 0.0                            # invalid: sum <= 0
    o = o.copy()
    bad = np.broadcast_to((np.arange(W)[:, None, None] != keep[None]), (W, T, H))
    o[bad] = 0x7fc0                                      # NaN payload in the invalid ones
    fo, fl = cp.cp_pack_permute_combine_fused(dev_payload(o, "bf16"), dev_f32(m), dev_f32(s))
    pkt, pl = cp.cp_pack_lse(dev_payload(o, "bf16"), dev_f32(m), dev_f32(s))
    torch.cuda.synchronize()
    got = host_bits(fo)                                   # [W, T, Hc, D]
    Hc = H // W
    t, h = np.meshgrid(np.arange(T), np.arange(H), indexing="ij")
    want = o[keep, t, h]                                  # [T, H, D]
    assert np.array_equal(got[h // Hc, t, h % Hc], want)
    lse_pkt = pl.cpu().numpy()                            # [W_src, W_dst, T, Hc]
    assert np.array_equal(fl.cpu().numpy()[h // Hc, t, h % Hc],
                          lse_pkt[keep, h // Hc, t, h % Hc])


def test_all_invalid_rows():
    W, T, H, D = 4, 33, 8, 64
    wl = synth.Workload("dead", W=W, T=T, H=H, D=D, seed=9)
    o, m, s = synth.full_inputs(wl)
    m = m.copy()
    m[:, 5, :] = np.nan
    m[:, 17, 3] = -np.inf
    fo, fl = cp.cp_pack_permute_combine_fused(dev_payload(o, "bf16"), dev_f32(m), dev_f32(s))
    torch.cuda.synchronize()
    Hc = H // W
    got, gl = host_bits(fo), fl.cpu().numpy()
    assert np.all(got[:, 5] == 0) and np.all(np.isneginf(gl[:, 5]))
    assert np.all(got[3 // Hc, 17, 3 % Hc] == 0) and np.isneginf(gl[3 // Hc, 17, 3 % Hc])
    assert np.isfinite(gl[:, 6]).all()


def test_ulysses_round_trip_config():
    wl = synth.CONFIGS["ulysses"]
    x = torch.randint(-32768, 32767, (wl.W, 3, wl.T // wl.W, wl.H, wl.D), dtype=torch.int16,
                      device="cuda").view(torch.bfloat16)
    y = cp.ulysses_seq2head(x)
    assert y.shape == (wl.W, 3, wl.T, wl.Hc, wl.D)
    z = cp.ulysses_head2seq(y)
    torch.cuda.synchronize()
    assert torch.equal(z.view(torch.int16), x.view(torch.int16))


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_legacy_pipeline_equals_max_sum_pack(name):
    """Materialize LSE, then pack from it (the Before pipeline) gives the packet of
    the max/sum-aware pack (the After pipeline) bit for bit."""
    wl = synth.CONFIGS[name]
    o, m, s = synth.full_inputs(wl)
    do, dm, ds = dev_payload(o, wl.dtype), dev_f32(m), dev_f32(s)
    for sd in (1, 0):
        a_o, a_l = cp.cp_pack_lse(do, dm, ds, scatter_dim=sd)
        lse = cp.cp_lse_materialize(dm, ds)
        b_o, b_l = cp.cp_pack_from_lse(do, lse, scatter_dim=sd)
        torch.cuda.synchronize()
        assert torch.equal(_bits(a_o), _bits(b_o))
        assert torch.equal(_bits(a_l), _bits(b_l))
