"""GPU path vs the CPU oracle, element by element, through the C-ABI.

Sizes are ones the oracle finishes in seconds, chosen to span several 32-row
chunks with ragged tails, every lanes-per-row shape (D = 8 ... 1024), W from 1
to 32, both payload types, strided inputs and the invalid-statistic patterns
of the workloads (NaN max, +inf sum, zero sum, +/-inf max, whole invalid
tokens). Payload and layout results must be bit-exact; LSE and combined
outputs meet the tolerances in ``gpu_util``.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import (FMT, check_combined, check_pack_lse, dev_f32, dev_payload, host_bits,
                      lse_member_tol)

pytestmark = pytest.mark.gpu

cp = pytest.importorskip("lse_pack_stable_b200")


def _wl(name, W, T, H, D, dtype="bf16", seed=11, **kw):
    base = dict(o_sigma=1.0, max_sigma=5.0, sum_dist=(synth.UNIFORM, 1.0, 256.0), p_invalid=0.03)
    base.update(kw)
    return synth.Workload(name, W=W, T=T, H=H, D=D, dtype=dtype, seed=seed, **base)


CASES = [
    synth.CONFIGS["tiny"],
    synth.CONFIGS["decode"],
    _wl("ragged_w3_d24", 3, 37, 6, 24),
    _wl("w5_d72_fp16", 5, 11, 10, 72, dtype="fp16"),
    _wl("w32_max", 32, 7, 64, 64),
    _wl("d1024_max", 2, 5, 4, 1024),
    _wl("d8_min", 4, 9, 4, 8),
    _wl("w1", 1, 13, 3, 16),
    _wl("w16_stress_like", 16, 40, 32, 128, dtype="fp16", o_sigma=2.0, max_sigma=10.0,
        sum_dist=(synth.LOGUNIFORM, 1e-3, 1e6), p_invalid=0.0, p_max_inf=0.05, p_sum_zero=0.05),
    _wl("w8_mla_like", 8, 24, 16, 512, o_sigma=0.5, max_sigma=8.0,
        sum_dist=(synth.LOGUNIFORM, 1.0, 1e5), p_invalid=0.01, p_token_invalid=0.1,
        last_token_invalid=True),
    _wl("w7_d40", 7, 19, 14, 40, dtype="fp16", p_invalid=0.2),
    _wl("w4_d256_many_invalid", 4, 33, 8, 256, p_invalid=0.6),
    # the widest register-staged rows (four 16-byte vectors per lane, ranks in
    # batches of four): D = 1024 at W = 8 and at W = 32; and the largest
    # shared-memory ring, D = 256 at W = 8 (one vector per lane, 32 lanes)
    _wl("w8_d1024_ring_max", 8, 5, 16, 1024, p_invalid=0.1),
    _wl("w8_d256_ring", 8, 9, 16, 256, p_invalid=0.1),
    _wl("w32_d1024_max", 32, 2, 32, 1024, p_invalid=0.1),
]
IDS = [c.name for c in CASES]

# Token-chunk exchange: destination j combines tokens j*T/W .. of every rank,
# all heads; the output is [T][H] in source order. T is a multiple of W here.
TOKEN_CASES = [
    synth.CONFIGS["tiny"],
    _wl("tok_w3_d24", 3, 36, 6, 24),
    _wl("tok_w5_d72_fp16", 5, 10, 10, 72, dtype="fp16"),
    _wl("tok_w32_max", 32, 64, 32, 64),
    _wl("tok_d1024", 2, 6, 4, 1024),
    _wl("tok_d8", 4, 12, 4, 8),
    _wl("tok_w1", 1, 13, 3, 16),
    _wl("tok_w16_stress_like", 16, 48, 32, 128, dtype="fp16", o_sigma=2.0, max_sigma=10.0,
        sum_dist=(synth.LOGUNIFORM, 1e-3, 1e6), p_invalid=0.0, p_max_inf=0.05, p_sum_zero=0.05),
    _wl("tok_w8_mla_like", 8, 24, 16, 512, o_sigma=0.5, max_sigma=8.0,
        sum_dist=(synth.LOGUNIFORM, 1.0, 1e5), p_invalid=0.01, p_token_invalid=0.1,
        last_token_invalid=True),
    _wl("tok_w7_d40", 7, 21, 14, 40, dtype="fp16", p_invalid=0.2),
    _wl("tok_w4_d256_many_invalid", 4, 36, 8, 256, p_invalid=0.6),
    _wl("tok_w8_d1024", 8, 8, 16, 1024, p_invalid=0.1),
]


def _scatter_params(cases, token_cases=TOKEN_CASES):
    """(workload, scatter_dim) pairs: head chunks for `cases`, token chunks for
    those of them with T % W == 0 and for `token_cases`."""
    seen, out = set(), []
    for sd in (1, 0):
        for wl in cases + (token_cases if sd == 0 else []):
            if (sd == 0 and wl.T % wl.W) or (wl.name, sd) in seen:
                continue
            seen.add((wl.name, sd))
            out.append(pytest.param(wl, sd, id="%s-sd%d" % (wl.name, sd)))
    return out


@pytest.fixture(scope="module")
def inputs():
    cache = {}

    def get(wl):
        if wl.name not in cache:
            o, m, s = synth.full_inputs(wl)
            cache[wl.name] = (o, m, s)
        return cache[wl.name]
    return get


def _dev_inputs(wl, o, m, s):
    return dev_payload(o, wl.dtype), dev_f32(m), dev_f32(s)


def _packet_layout(a, W, T, H, scatter_dim):
    if scatter_dim == 1:
        return a.reshape(W, T, W, H // W).transpose(0, 2, 1, 3)
    return a.reshape(W, W, T // W, H)


# ------------------------------------------------------------------------------------ pack

@pytest.mark.parametrize("wl,scatter_dim", _scatter_params(CASES))
def test_pack(wl, scatter_dim, inputs, orc):
    o, m, s = inputs(wl)
    do, dm, ds = _dev_inputs(wl, o, m, s)
    pkt, pl = cp.cp_pack_lse(do, dm, ds, scatter_dim=scatter_dim)
    torch.cuda.synchronize()
    ref_o, _, ref_l = orc.pack(o, m, s, scatter_dim)
    assert np.array_equal(host_bits(pkt), ref_o), "packet payload differs"
    W, T, H = wl.W, wl.T, wl.H
    check_pack_lse(pl.cpu().numpy(), ref_l, _packet_layout(m, W, T, H, scatter_dim),
                   _packet_layout(s, W, T, H, scatter_dim))


def test_pack_strided_inputs(orc):
    wl = _wl("strided", 4, 21, 8, 64, p_invalid=0.05)
    o, m, s = synth.full_inputs(wl)
    W, T, H, D = o.shape
    # padded parents: gaps between heads, tokens and ranks; stats interleaved
    big = torch.zeros((W + 1, T + 3, H + 2, D + 16), dtype=torch.bfloat16, device="cuda")
    ov = big[1:, 2:T + 2, 1:H + 1, 8:D + 8]
    ov.copy_(dev_payload(o, "bf16"))
    bm = torch.zeros((W, T, 3 * H), dtype=torch.float32, device="cuda")
    mv = bm[:, :, 1::3]
    mv.copy_(dev_f32(m))
    sv = dev_f32(s).transpose(0, 1).contiguous().transpose(0, 1)   # [W,T,H] view, t-major storage
    assert not ov.is_contiguous() and not mv.is_contiguous() and not sv.is_contiguous()
    pkt, pl = cp.cp_pack_lse(ov, mv, sv, scatter_dim=1)
    fo, fl = cp.cp_pack_permute_combine_fused(ov, mv, sv)
    torch.cuda.synchronize()
    ref_o, _, ref_l = orc.pack(o, m, s, 1)
    assert np.array_equal(host_bits(pkt), ref_o)
    check_pack_lse(pl.cpu().numpy(), ref_l, _packet_layout(m, W, T, H, 1),
                   _packet_layout(s, W, T, H, 1))
    ref, ref_lse, ref_r = orc.fused(o, m, s, FMT["bf16"])
    check_combined(host_bits(fo), fl.cpu().numpy(), ref, ref_lse, ref_r, "bf16", W,
                   extra_lse_tol=lse_member_tol(m.reshape(W, -1), s.reshape(W, -1)).reshape(
                       T, W, H // W).transpose(1, 0, 2))
    # and the contiguous inputs give the same bits
    co, cl = cp.cp_pack_permute_combine_fused(*_dev_inputs(wl, o, m, s))
    assert torch.equal(co.view(torch.int16), fo.view(torch.int16))
    assert torch.equal(cl.view(torch.int32), fl.view(torch.int32))


@pytest.mark.parametrize("scatter_dim", [1, 0])
def test_pack_block_copy_padded_token_stride(scatter_dim, orc):
    """Heads back to back within a token (so_h == D), gaps between tokens and
    between ranks: the block-copy pack for head and for token chunks, its
    legacy twin, and the per-rank pack of one such plane, against the oracle."""
    wl = _wl("padded_tokens", 4, 20, 8, 64, p_invalid=0.05)
    o, m, s = synth.full_inputs(wl)
    W, T, H, D = o.shape
    row = H * D + 64                                   # token stride: 64 elements of padding
    big = torch.zeros((W + 1) * (T + 3) * row, dtype=torch.bfloat16, device="cuda")
    ov = torch.as_strided(big, (W, T, H, D), ((T + 3) * row, row, D, 1), storage_offset=row + 8)
    ov.copy_(dev_payload(o, "bf16"))
    assert ov.stride(2) == D and ov.stride(1) != H * D
    dm, ds = dev_f32(m), dev_f32(s)
    pkt, pl = cp.cp_pack_lse(ov, dm, ds, scatter_dim=scatter_dim)
    lse = cp.cp_lse_materialize(dm, ds)
    lpkt, lpl = cp.cp_pack_from_lse(ov, lse, scatter_dim=scatter_dim)
    r = 2
    rpkt, rpl = cp.cp_pack_lse_rank(ov[r], dm[r], ds[r], W, scatter_dim=scatter_dim)
    torch.cuda.synchronize()
    ref_o, _, ref_l = orc.pack(o, m, s, scatter_dim)
    assert np.array_equal(host_bits(pkt), ref_o), "packet payload differs"
    check_pack_lse(pl.cpu().numpy(), ref_l, _packet_layout(m, W, T, H, scatter_dim),
                   _packet_layout(s, W, T, H, scatter_dim))
    assert torch.equal(lpkt.view(torch.int16), pkt.view(torch.int16))
    assert torch.equal(rpkt.view(torch.int16), pkt[r].view(torch.int16))
    assert torch.equal(rpl.view(torch.int32), pl[r].view(torch.int32))


# ------------------------------------------------------------------------------------ permute

@pytest.mark.parametrize("W,block_bytes", [(1, 48), (2, 16), (4, 4096), (5, 3), (8, 1000),
                                           (3, 18), (16, 64), (32, 32),
                                           # several grid tiles per block plus a ragged tail
                                           (6, 3 * 32768 + 24), (32, 4104)])
def test_permute_blocks(W, block_bytes, orc):
    rng = np.random.default_rng(W * 1000 + block_bytes)
    send = rng.integers(0, 256, size=W * W * block_bytes, dtype=np.uint8)
    recv = cp.cp_a2a_local_permute(torch.from_numpy(send).cuda(), W)
    torch.cuda.synchronize()
    assert np.array_equal(recv.cpu().numpy(), orc.permute(send, W))


@pytest.mark.parametrize("wl", CASES[:4], ids=IDS[:4])
def test_permute_packet_regions(wl, inputs, orc):
    o, m, s = inputs(wl)
    pkt, l32, _ = orc.pack(o, m, s, 1)
    g_o = cp.cp_a2a_local_permute(dev_payload(pkt, wl.dtype), wl.W)
    g_l = cp.cp_a2a_local_permute(dev_f32(l32), wl.W)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(g_o), orc.permute(pkt, wl.W))
    assert np.array_equal(g_l.cpu().numpy().view(np.uint32), orc.permute(l32, wl.W).view(np.uint32))


# ------------------------------------------------------------------------------------ combine

@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_combine_received_packet(wl, inputs, orc):
    """The combine on the oracle's own packet, after the oracle's all-to-all."""
    o, m, s = inputs(wl)
    pkt, l32, _ = orc.pack(o, m, s, 1)
    recv_o, recv_l = orc.permute(pkt, wl.W), orc.permute(l32, wl.W)
    out, out_lse = cp.cp_lse_combine(dev_payload(recv_o, wl.dtype), dev_f32(recv_l))
    torch.cuda.synchronize()
    ref, ref_lse, ref_r = orc.combine(recv_o, recv_l, FMT[wl.dtype])
    check_combined(host_bits(out), out_lse.cpu().numpy(), ref, ref_lse, ref_r, wl.dtype, wl.W)


@pytest.mark.parametrize("W,T,Hc,D,dtype,p_dead", [(4, 50, 3, 128, "bf16", 0.3),
                                                   (8, 17, 2, 512, "fp16", 0.5),
                                                   (2, 64, 4, 64, "bf16", 0.0),
                                                   (16, 9, 1, 8, "bf16", 0.9),
                                                   (32, 5, 2, 136, "fp16", 0.2)])
def test_combine_direct_lse(W, T, Hc, D, dtype, p_dead, orc):
    """Received LSE drawn directly (wide N(0, 6) spread and -inf holes, NaN too)."""
    wl = _wl("direct", W, T, Hc * W, D, dtype=dtype, seed=W + D)
    N = T * Hc
    lse = synth.received_lse(wl, p_dead, W * N).reshape(W, W, T, Hc)
    lse.reshape(-1)[::97] = np.nan                      # NaN counts as invalid
    bits = synth.fill(wl.seed, synth.TID_O, synth.NORMAL, 0.0, 1.0, n=W * W * N * D,
                      fmt=synth.BF16 if dtype == "bf16" else synth.F16).reshape(W, W, T, Hc, D)
    bits = bits.copy()
    # invalid contributions carry NaN payload, which must not reach the output
    nan_bits = 0x7fc0 if dtype == "bf16" else 0x7e00
    bits[~(lse > -np.inf)] = nan_bits
    out, out_lse = cp.cp_lse_combine(dev_payload(bits, dtype), dev_f32(lse))
    torch.cuda.synchronize()
    ref, ref_lse, ref_r = orc.combine(bits, lse, FMT[dtype])
    check_combined(host_bits(out), out_lse.cpu().numpy(), ref, ref_lse, ref_r, dtype, W)


# ------------------------------------------------------------------------------------ fused

@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_fused(wl, inputs, orc):
    o, m, s = inputs(wl)
    out, out_lse = cp.cp_pack_permute_combine_fused(*_dev_inputs(wl, o, m, s))
    torch.cuda.synchronize()
    ref, ref_lse, ref_r = orc.fused(o, m, s, FMT[wl.dtype])
    W, T, H = wl.W, wl.T, wl.H
    extra = lse_member_tol(m.reshape(W, -1), s.reshape(W, -1)).reshape(T, W, H // W).transpose(1, 0, 2)
    check_combined(host_bits(out), out_lse.cpu().numpy(), ref, ref_lse, ref_r, wl.dtype, W,
                   extra_lse_tol=extra)


@pytest.mark.parametrize("wl", TOKEN_CASES, ids=[c.name for c in TOKEN_CASES])
def test_fused_token_scatter(wl, inputs, orc):
    o, m, s = inputs(wl)
    W, T, H, D = wl.W, wl.T, wl.H, wl.D
    do, dm, ds = _dev_inputs(wl, o, m, s)
    out, out_lse = cp.cp_pack_permute_combine_fused(do, dm, ds, scatter_dim=0)
    assert out.shape == (W, T // W, H, D) and out_lse.shape == (W, T // W, H)
    # the unfused token-chunk chain, bit for bit
    pkt, pl = cp.cp_pack_lse(do, dm, ds, scatter_dim=0)
    co, cl = cp.cp_lse_combine(cp.cp_a2a_local_permute(pkt, W), cp.cp_a2a_local_permute(pl, W))
    torch.cuda.synchronize()
    assert torch.equal(co.view(torch.int16), out.view(torch.int16))
    assert torch.equal(cl.view(torch.int32), out_lse.view(torch.int32))
    # against the oracle's direct merge of every (t, h), in source order
    ref, ref_lse, ref_r = orc.fused_gathered(o.reshape(W, T * H, D), m.reshape(W, T * H),
                                             s.reshape(W, T * H), FMT[wl.dtype])
    check_combined(host_bits(out).reshape(T * H, D), out_lse.cpu().numpy().reshape(-1), ref,
                   ref_lse, ref_r, wl.dtype, W,
                   extra_lse_tol=lse_member_tol(m.reshape(W, -1), s.reshape(W, -1)))


def test_fused_token_scatter_strided_inputs(orc):
    wl = _wl("tok_strided", 4, 24, 8, 64, p_invalid=0.05)
    o, m, s = synth.full_inputs(wl)
    W, T, H, D = o.shape
    big = torch.zeros((W + 1, T + 3, H + 2, D + 16), dtype=torch.bfloat16, device="cuda")
    ov = big[1:, 2:T + 2, 1:H + 1, 8:D + 8]
    ov.copy_(dev_payload(o, "bf16"))
    bm = torch.zeros((W, T, 3 * H), dtype=torch.float32, device="cuda")
    mv = bm[:, :, 1::3]
    mv.copy_(dev_f32(m))
    sv = dev_f32(s).transpose(0, 1).contiguous().transpose(0, 1)
    fo, fl = cp.cp_pack_permute_combine_fused(ov, mv, sv, scatter_dim=0)
    co, cl = cp.cp_pack_permute_combine_fused(*_dev_inputs(wl, o, m, s), scatter_dim=0)
    torch.cuda.synchronize()
    assert torch.equal(co.view(torch.int16), fo.view(torch.int16))
    assert torch.equal(cl.view(torch.int32), fl.view(torch.int32))
    ref, ref_lse, ref_r = orc.fused_gathered(o.reshape(W, T * H, D), m.reshape(W, T * H),
                                             s.reshape(W, T * H), FMT["bf16"])
    check_combined(host_bits(fo).reshape(T * H, D), fl.cpu().numpy().reshape(-1), ref, ref_lse,
                   ref_r, "bf16", W, extra_lse_tol=lse_member_tol(m.reshape(W, -1), s.reshape(W, -1)))


# ------------------------------------------------------------------------------------ Ulysses

ULY = [(2, 3, 4, 4, 8, 2), (4, 1, 3, 8, 128, 2), (3, 2, 5, 6, 24, 2), (8, 3, 16, 48, 128, 2),
       (1, 2, 3, 2, 64, 2), (4, 2, 3, 4, 3, 1), (2, 1, 5, 2, 5, 4), (4, 1, 2, 4, 7, 8),
       (8, 1, 64, 8, 128, 2)]


@pytest.mark.parametrize("W,B,S_l,H,D,eb", ULY)
def test_ulysses(W, B, S_l, H, D, eb, orc):
    rng = np.random.default_rng(W * 7 + D)
    npdt = {1: np.uint8, 2: np.uint16, 4: np.uint32, 8: np.uint64}[eb]
    tdt = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}[eb]
    x = rng.integers(0, 2 ** (8 * eb) - 1, size=(W, B, S_l, H, D), dtype=npdt)
    xd = torch.from_numpy(x.view({1: np.uint8, 2: np.int16, 4: np.int32, 8: np.int64}[eb])).cuda()
    assert xd.dtype == tdt
    y = cp.ulysses_seq2head(xd)
    back = cp.ulysses_head2seq(y)
    z = rng.integers(0, 2 ** (8 * eb) - 1, size=(W, B, S_l * W, H // W, D), dtype=npdt)
    zd = torch.from_numpy(z.view(xd.cpu().numpy().dtype)).cuda()
    w = cp.ulysses_head2seq(zd)
    torch.cuda.synchronize()
    view = lambda t: t.cpu().numpy().view(npdt)
    assert np.array_equal(view(y), orc.seq2head(x))
    assert np.array_equal(view(back), x)
    assert np.array_equal(view(w), orc.head2seq(z))


@pytest.mark.parametrize("W,B,S_l,H,D,eb", [(2, 65537, 1, 2, 4, 2), (4, 70001, 1, 4, 3, 1),
                                              (2, 65600, 2, 2, 8, 4)])
def test_ulysses_many_batch_planes(W, B, S_l, H, D, eb, orc):
    """More batch planes than one grid dimension holds (B > 65535): the
    one-warp-per-chunk launch, both directions, against the oracle."""
    rng = np.random.default_rng(B)
    npdt = {1: np.uint8, 2: np.uint16, 4: np.uint32}[eb]
    sdt = {1: np.uint8, 2: np.int16, 4: np.int32}[eb]
    x = rng.integers(0, 2 ** (8 * eb) - 1, size=(W, B, S_l, H, D), dtype=npdt)
    y = cp.ulysses_seq2head(torch.from_numpy(x.view(sdt)).cuda())
    back = cp.ulysses_head2seq(y)
    torch.cuda.synchronize()
    view = lambda t: t.cpu().numpy().view(npdt)
    assert np.array_equal(view(y), orc.seq2head(x))
    assert np.array_equal(view(back), x)


# ------------------------------------------------------------------------------------ edges

def test_empty_inputs_are_noops():
    e = torch.empty((2, 0, 4, 64), dtype=torch.bfloat16, device="cuda")
    st = torch.empty((2, 0, 4), dtype=torch.float32, device="cuda")
    out, lse = cp.cp_pack_permute_combine_fused(e, st, st)
    pkt, pl = cp.cp_pack_lse(e, st, st)
    o2, l2 = cp.cp_lse_combine(pkt, pl)
    assert out.numel() == 0 and pkt.numel() == 0 and o2.numel() == 0
    x = torch.empty((2, 0, 3, 4, 8), dtype=torch.bfloat16, device="cuda")
    assert cp.ulysses_seq2head(x).numel() == 0
    assert cp.cp_a2a_local_permute(torch.empty(0, device="cuda"), 4).numel() == 0


def _guarded(shape, dtype, pad=4096):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * pad,), 0x5A5A if dtype != torch.float32 else 0,
                     dtype=torch.int16 if dtype != torch.float32 else torch.int32, device="cuda")
    if dtype == torch.float32:
        buf.fill_(0x5A5A5A5A)
        inner = buf[pad:pad + n].view(torch.float32).view(shape)
    else:
        inner = buf[pad:pad + n].view(dtype).view(shape)
    return buf, inner, pad, n


def _canary_ok(buf, pad, n):
    v = buf.cpu().numpy()
    want = 0x5A5A if buf.dtype == torch.int16 else 0x5A5A5A5A
    return np.all(v[:pad] == want) and np.all(v[pad + n:] == want)


@pytest.mark.parametrize("wl", [CASES[2], CASES[3], CASES[8]], ids=[IDS[2], IDS[3], IDS[8]])
def test_outputs_stay_in_bounds(wl, inputs):
    """Canary bands around every output survive pack, permute, combine and fused."""
    o, m, s = inputs(wl)
    do, dm, ds = _dev_inputs(wl, o, m, s)
    W, T, H, D = wl.W, wl.T, wl.H, wl.D
    tdt = do.dtype
    b1, pkt, p1, n1 = _guarded((W, W, T, H // W, D), tdt)
    b2, pl, p2, n2 = _guarded((W, W, T, H // W), torch.float32)
    cp.cp_pack_lse(do, dm, ds, pkt_o=pkt, pkt_lse=pl)
    b3, rcv, p3, n3 = _guarded((W, W, T, H // W, D), tdt)
    b4, rl, p4, n4 = _guarded((W, W, T, H // W), torch.float32)
    cp.cp_a2a_local_permute(pkt, W, recv=rcv)
    cp.cp_a2a_local_permute(pl, W, recv=rl)
    b5, out, p5, n5 = _guarded((W, T, H // W, D), tdt)
    b6, ol, p6, n6 = _guarded((W, T, H // W), torch.float32)
    cp.cp_lse_combine(rcv, rl, out=out, out_lse=ol)
    b7, fo, p7, n7 = _guarded((W, T, H // W, D), tdt)
    b8, fl, p8, n8 = _guarded((W, T, H // W), torch.float32)
    cp.cp_pack_permute_combine_fused(do, dm, ds, out=fo, out_lse=fl)
    x = torch.randint(-30000, 30000, (W, 2, 3, H, D), dtype=torch.int16, device="cuda")
    b9, y, p9, n9 = _guarded((W, 2, 3 * W, H // W, D), torch.int16)
    cp.ulysses_seq2head(x, out=y)
    torch.cuda.synchronize()
    for b, p, n in [(b1, p1, n1), (b2, p2, n2), (b3, p3, n3), (b4, p4, n4), (b5, p5, n5),
                    (b6, p6, n6), (b7, p7, n7), (b8, p8, n8), (b9, p9, n9)]:
        assert _canary_ok(b, p, n)


# ------------------------------------------------------------------------------------ legacy

@pytest.mark.parametrize("wl", [CASES[0], CASES[1], CASES[3], CASES[8], CASES[10]],
                         ids=[IDS[0], IDS[1], IDS[3], IDS[8], IDS[10]])
def test_lse_materialize(wl, inputs, orc):
    """Legacy first step: the standalone LSE tensor, 2 ulp of the float64 LSE."""
    _, m, s = inputs(wl)
    lse = cp.cp_lse_materialize(dev_f32(m), dev_f32(s))
    torch.cuda.synchronize()
    check_pack_lse(lse.cpu().numpy(), orc.materialize_lse(m, s), m, s)


def test_lse_materialize_strided(orc):
    wl = _wl("strided_stats", 3, 17, 6, 8, p_invalid=0.1)
    _, m, s = synth.full_inputs(wl)
    bm = torch.zeros((3, 17, 12), dtype=torch.float32, device="cuda")
    bm[:, :, 1::2] = dev_f32(m)
    sv = dev_f32(s).transpose(0, 1).contiguous().transpose(0, 1)
    lse = cp.cp_lse_materialize(bm[:, :, 1::2], sv)
    torch.cuda.synchronize()
    check_pack_lse(lse.cpu().numpy(), orc.materialize_lse(m, s), m, s)


@pytest.mark.parametrize("wl,scatter_dim", _scatter_params(
    [CASES[0], CASES[2], CASES[4], CASES[6], CASES[9]],
    token_cases=[TOKEN_CASES[1], TOKEN_CASES[3], TOKEN_CASES[5]]))
def test_pack_from_lse(wl, scatter_dim, inputs, orc):
    """Legacy pack: payload and the materialized LSE moved into the packet, bit-exact."""
    o, _, _ = inputs(wl)
    lse = synth.received_lse(wl, 0.1, wl.T * wl.H).reshape(wl.W, wl.T, wl.H)
    pkt, pl = cp.cp_pack_from_lse(dev_payload(o, wl.dtype), dev_f32(lse), scatter_dim=scatter_dim)
    torch.cuda.synchronize()
    ref_o, ref_l = orc.pack_from_lse(o, lse, scatter_dim)
    assert np.array_equal(host_bits(pkt), ref_o)
    assert np.array_equal(pl.cpu().numpy().view(np.uint32), ref_l.view(np.uint32))
