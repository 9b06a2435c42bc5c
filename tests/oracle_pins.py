"""Pins of the CPU oracle to facts outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises ``AssertionError``
when the oracle disagrees with something the pages or mathematics fix:
hand-derived closed forms (``golden/``), library routines that compute the same
quantity another way (scipy's logsumexp/softmax for brute-force attention,
numpy and torch for the 16-bit formats, numpy split/concatenate and transposes
for the layout maps), and invariants of the combine. ``test_oracle.py`` runs
them on the oracle; ``test_oracle_mutants.py`` runs them on copies of the
oracle with planted mistakes and expects each mistake to be caught.
"""
from __future__ import annotations

import math
import os

import numpy as np
import scipy.special
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
BF16, FP16 = 0, 1


def _num(tok: str) -> float:
    return float(tok)


def read_lse_cases():
    rows = []
    with open(os.path.join(GOLDEN, "lse_formation.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                m, s, e = line.split()
                rows.append((_num(m), _num(s), _num(e)))
    return rows


def read_combine_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "combine_closed_forms.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "case":
                cur = {"name": vals[0], "o": []}
                cases.append(cur)
            elif key == "o":
                cur["o"].append([_num(v) for v in vals])
            else:
                cur[key] = [_num(v) for v in vals]
    return cases


def _close(a: float, b: float, rel: float = 1e-15) -> bool:
    if math.isinf(b) or math.isinf(a):
        return a == b
    return abs(a - b) <= rel * max(1.0, abs(b))


# ---------------------------------------------------------------------------- LSE formation

def pin_lse_golden(orc):
    """Invalid-statistic rule and closed-form LSE values (golden/lse_formation.txt)."""
    for m, s, expect in read_lse_cases():
        got = orc.lse(np.float32(m), np.float32(s))
        assert _close(got, expect), (m, s, got, expect)


# ---------------------------------------------------------------------------- combine

def pin_combine_golden(orc):
    """Hand-derived closed forms (golden/combine_closed_forms.txt)."""
    for c in read_combine_cases():
        o = np.array(c["o"], dtype=np.float64)[:, None, :]       # [W, 1, D]
        lse = np.array(c["lse"], dtype=np.float64)[:, None]       # [W, 1]
        out, out_lse = orc.combine_f64(o, lse)
        assert _close(out_lse[0], c["expect_lse"][0]), (c["name"], out_lse[0])
        for g, e in zip(out[0], c["expect_o"]):
            assert _close(g, e, 1e-14), (c["name"], out[0], c["expect_o"])


def _attention_partials(rng, W, n_keys, n_q, Dk, D, empty_shard=True):
    """Brute-force softmax attention: full result and per-KV-shard partials."""
    q = rng.standard_normal((n_q, Dk))
    K = rng.standard_normal((n_keys, Dk))
    V = rng.standard_normal((n_keys, D))
    scores = q @ K.T / math.sqrt(Dk)                           # [n_q, n_keys]
    full_o = scipy.special.softmax(scores, axis=1) @ V
    full_lse = scipy.special.logsumexp(scores, axis=1)
    # uneven contiguous shards, one of them empty
    cuts = np.sort(rng.choice(np.arange(1, n_keys), size=W - 1, replace=False))
    if empty_shard and W >= 3:
        cuts[1] = cuts[0]
    bounds = [0, *cuts.tolist(), n_keys]
    o_r = np.full((W, n_q, D), np.nan)
    m_r = np.full((W, n_q), -np.inf)
    s_r = np.zeros((W, n_q))
    shard_lse = np.full((W, n_q), -np.inf)
    for r in range(W):
        a, b = bounds[r], bounds[r + 1]
        if a == b:
            continue                                           # empty: max -inf, sum 0
        sc = scores[:, a:b]
        m_r[r] = sc.max(axis=1)
        p = np.exp(sc - m_r[r][:, None])
        s_r[r] = p.sum(axis=1)
        o_r[r] = (p @ V[a:b]) / s_r[r][:, None]
        shard_lse[r] = scipy.special.logsumexp(sc, axis=1)
    return full_o, full_lse, o_r, m_r, s_r, shard_lse


def pin_bruteforce_attention(orc):
    """Softmax attention over the full KV set equals the combine of the per-shard
    partial attentions, with each partial's LSE formed from its own (max, sum);
    one shard is empty (max -inf, sum 0: invalid) and carries NaN payload."""
    rng = np.random.default_rng(20260913)
    for W, n_keys in [(2, 9), (3, 17), (4, 40), (7, 33)]:
        full_o, full_lse, o_r, m_r, s_r, shard_lse = _attention_partials(
            rng, W, n_keys, n_q=5, Dk=16, D=12)
        lse = np.vectorize(orc.lse)(m_r, s_r)
        fin = np.isfinite(shard_lse)
        assert np.array_equal(np.isfinite(lse), fin)
        assert np.allclose(lse[fin], shard_lse[fin], rtol=0, atol=1e-12)
        out, out_lse = orc.combine_f64(o_r, lse)
        assert np.allclose(out, full_o, rtol=0, atol=1e-12), np.abs(out - full_o).max()
        assert np.allclose(out_lse, full_lse, rtol=0, atol=1e-12)


def pin_combine_invariants(orc):
    rng = np.random.default_rng(7)
    W, N, D = 5, 64, 24
    o = rng.standard_normal((W, N, D))
    lse = rng.normal(0, 6, (W, N))
    lse[rng.random((W, N)) < 0.2] = -np.inf
    lse[:, 3] = -np.inf                                        # an all-invalid row
    out, out_lse = orc.combine_f64(o, lse)
    # all-invalid row: exactly +0 and -inf
    assert np.all(out[3] == 0) and not np.any(np.signbit(out[3])) and out_lse[3] == -np.inf
    # shift invariance
    out2, lse2 = orc.combine_f64(o, lse + 3.75)
    ok = np.isfinite(out_lse)
    assert np.allclose(out2, out, rtol=0, atol=1e-12)
    assert np.allclose(lse2[ok], out_lse[ok] + 3.75, rtol=0, atol=1e-12)
    # permutation of the contributions
    perm = rng.permutation(W)
    out3, lse3 = orc.combine_f64(o[perm], lse[perm])
    assert np.allclose(out3, out, rtol=0, atol=1e-12)
    assert np.allclose(lse3[ok], out_lse[ok], rtol=0, atol=1e-12)
    # convexity: componentwise between the min and max of the valid contributions
    valid = np.isfinite(lse)
    hi = np.where(valid[:, :, None], o, -np.inf).max(axis=0)
    lo = np.where(valid[:, :, None], o, np.inf).min(axis=0)
    assert np.all(out[ok] <= hi[ok] + 1e-12) and np.all(out[ok] >= lo[ok] - 1e-12)
    # W = 1 is the identity, bit for bit
    one, one_lse = orc.combine_f64(o[:1], lse[:1])
    f = np.isfinite(lse[0])
    assert np.array_equal(one[f], o[0][f]) and np.array_equal(one_lse[f], lse[0][f])
    # a single valid contribution comes through exactly, whatever the others carry
    lse1 = np.full((W, N), -np.inf)
    lse1[2] = lse[2]
    o_nan = o.copy()
    o_nan[[0, 1, 3, 4]] = np.nan
    s_out, s_lse = orc.combine_f64(o_nan, lse1)
    f = np.isfinite(lse[2])
    assert np.array_equal(s_out[f], o[2][f]) and np.array_equal(s_lse[f], lse[2][f])
    # two equal LSEs: the mean, LSE + ln 2
    lse_eq = np.tile(lse[:1], (2, 1))
    m_out, m_lse = orc.combine_f64(o[:2], lse_eq)
    f = np.isfinite(lse[0])
    assert np.allclose(m_out[f], 0.5 * (o[0][f] + o[1][f]), rtol=0, atol=1e-13)
    assert np.allclose(m_lse[f], lse[0][f] + 0.69314718055994531, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------- 16-bit formats

def pin_payload_formats(orc):
    """Decoding and nearest-even rounding of bf16 / fp16 against numpy and torch."""
    bits = np.arange(65536, dtype=np.uint16)
    ref16 = bits.view(np.float16).astype(np.float64)
    got16 = np.array([orc.payload_value(b, FP16) for b in bits])
    same = (got16 == ref16) | (np.isnan(got16) & np.isnan(ref16))
    assert same.all(), np.flatnonzero(~same)[:5]
    refbf = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    gotbf = np.array([orc.payload_value(b, BF16) for b in bits])
    same = (gotbf == refbf) | (np.isnan(gotbf) & np.isnan(refbf))
    assert same.all(), np.flatnonzero(~same)[:5]
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 6, 4000),
        ref16[np.isfinite(ref16)][::37] * (1 + 2.0 ** -11),    # just above fp16 midpoints
        [65504.0, 65519.9, 65520.0, 1e6, -1e6, 2.0 ** -25, 3 * 2.0 ** -26, 0.0, -0.0],
    ])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    got = np.array([orc.payload_round(v, FP16) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:5]
    xf = (rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000)).astype(np.float32)
    xf = np.concatenate([xf, np.float32([3.3895314e38, 1e-40, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8])])
    want = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.payload_round(float(v), BF16) for v in xf], dtype=np.uint16)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:5]


# ---------------------------------------------------------------------------- layouts

def _iota_inputs(W, T, H, D, seed=0):
    n = W * T * H * D
    assert n <= 65536
    o = np.arange(n, dtype=np.uint16).reshape(W, T, H, D)
    rng = np.random.default_rng(seed)
    mx = rng.standard_normal((W, T, H)).astype(np.float32)   # distinct values
    sm = np.ones((W, T, H), dtype=np.float32)                # log(1) = 0: LSE = max exactly
    return o, mx, sm


def pin_pack_layout(orc):
    """Head-chunk and token-chunk packets against numpy reshapes/transposes, on
    distinct (iota) payload bits; strided inputs give the same packet."""
    for W, T, H, D in [(2, 3, 4, 8), (4, 4, 8, 8), (3, 6, 6, 16), (1, 5, 3, 8)]:
        o, mx, sm = _iota_inputs(W, T, H, D)
        Hc = H // W
        pkt, l32, l64 = orc.pack(o, mx, sm, scatter_dim=1)
        want = o.reshape(W, T, W, Hc, D).transpose(0, 2, 1, 3, 4)
        assert np.array_equal(pkt, want)
        assert np.array_equal(l64, mx.reshape(W, T, W, Hc).transpose(0, 2, 1, 3).astype(np.float64))
        assert np.array_equal(l32, l64.astype(np.float32))
        if T % W == 0:
            pkt0, _, l0 = orc.pack(o, mx, sm, scatter_dim=0)
            assert np.array_equal(pkt0, o.reshape(W, W, T // W, H, D))
            assert np.array_equal(l0, mx.reshape(W, W, T // W, H).astype(np.float64))
        # strided: a padded parent array, views with gaps in every dimension
        big = np.zeros((W + 1, T + 2, H + 3, D + 8), dtype=np.uint16)
        big[1:, 1:T + 1, 2:H + 2, 4:D + 4] = o
        ov = big[1:, 1:T + 1, 2:H + 2, 4:D + 4]
        bm = np.zeros((W, T, 2 * H), dtype=np.float32)
        bm[:, :, ::2] = mx
        pkt_s, _, l64s = orc.pack(ov, bm[:, :, ::2], sm, scatter_dim=1)
        assert np.array_equal(pkt_s, pkt) and np.array_equal(l64s, l64)


def pin_pack_from_lse(orc):
    """Legacy pack: the LSE region is the materialized LSE moved by the same map
    as the payload (numpy reshape/transpose), bits unchanged, strided input too."""
    rng = np.random.default_rng(11)
    for W, T, H, D in [(2, 3, 4, 8), (4, 4, 8, 8), (3, 6, 6, 16)]:
        o, _, _ = _iota_inputs(W, T, H, D)
        lse = rng.standard_normal((W, T, H)).astype(np.float32)
        lse[0, 0, 0] = -np.inf
        Hc = H // W
        pkt, pl = orc.pack_from_lse(o, lse, 1)
        assert np.array_equal(pkt, o.reshape(W, T, W, Hc, D).transpose(0, 2, 1, 3, 4))
        assert np.array_equal(pl.view(np.uint32),
                              lse.reshape(W, T, W, Hc).transpose(0, 2, 1, 3).view(np.uint32))
        if T % W == 0:
            pkt0, pl0 = orc.pack_from_lse(o, lse, 0)
            assert np.array_equal(pl0, lse.reshape(W, W, T // W, H))
        big = np.zeros((W, T, 2 * H), dtype=np.float32)
        big[:, :, 1::2] = lse
        _, pls = orc.pack_from_lse(o, big[:, :, 1::2], 1)
        assert np.array_equal(pls, pl)


def pin_permute(orc):
    rng = np.random.default_rng(1)
    for W, blk in [(1, 24), (2, 8), (4, 12), (5, 3)]:
        send = rng.integers(0, 255, size=(W, W, blk), dtype=np.uint8)
        recv = orc.permute(send, W)
        assert np.array_equal(recv, send.swapaxes(0, 1))
        assert np.array_equal(orc.permute(recv, W), send)


def _uly_seq2head_np(x):
    W = x.shape[0]
    return np.stack([np.concatenate([np.split(x[r], W, axis=2)[j] for r in range(W)], axis=1)
                     for j in range(W)])


def _uly_head2seq_np(x):
    W = x.shape[0]
    return np.stack([np.concatenate([np.split(x[r], W, axis=1)[j] for r in range(W)], axis=2)
                     for j in range(W)])


def pin_ulysses(orc):
    """all_to_all_4D layouts as torch chunk/cat semantics (numpy split/concatenate),
    and head2seq(seq2head(x)) == x."""
    rng = np.random.default_rng(2)
    for W, B, S_l, H, D in [(2, 3, 4, 4, 8), (4, 1, 3, 8, 4), (3, 2, 5, 6, 2), (1, 2, 3, 2, 4)]:
        x = rng.integers(0, 65535, size=(W, B, S_l, H, D), dtype=np.uint16)
        y = orc.seq2head(x)
        assert np.array_equal(y, _uly_seq2head_np(x))
        assert np.array_equal(orc.head2seq(y), x)
        z = rng.integers(0, 65535, size=(W, B, S_l * W, H // W, D), dtype=np.uint16)
        assert np.array_equal(orc.head2seq(z), _uly_head2seq_np(z))


# ---------------------------------------------------------------------------- composition

def pin_fused_equals_chain(orc):
    """Direct merge == pack -> all-to-all -> combine on the oracle's own packet:
    exactly when every LSE is representable in float32 (sum = 1), and to float32
    rounding of the packet LSE otherwise."""
    rng = np.random.default_rng(5)
    for W, T, H, D, dt in [(2, 5, 4, 8, BF16), (4, 3, 8, 16, FP16), (3, 4, 6, 8, BF16)]:
        o = rng.integers(0, 65535, size=(W, T, H, D), dtype=np.uint16)
        o = np.where((o & 0x7f80) == 0x7f80, o & 0x3fff, o).astype(np.uint16)  # finite bf16
        if dt == FP16:
            o = np.where((o & 0x7c00) == 0x7c00, o & 0x3bff, o).astype(np.uint16)
        mx = rng.normal(0, 4, (W, T, H)).astype(np.float32)
        for exact in (True, False):
            sm = (np.ones((W, T, H)) if exact else rng.uniform(0.5, 50, (W, T, H))).astype(np.float32)
            sm[rng.random((W, T, H)) < 0.15] = 0.0
            f_out, f_lse, _ = orc.fused(o, mx, sm, dt)
            pkt, l32, _ = orc.pack(o, mx, sm, 1)
            recv = orc.permute(pkt, W)
            rl = orc.permute(l32, W)
            c_out, c_lse, _ = orc.combine(recv, rl, dt)
            if exact:
                assert np.array_equal(c_out, f_out) and np.array_equal(c_lse, f_lse)
            else:
                assert np.allclose(c_out, f_out, rtol=1e-5, atol=1e-5)
                fin = np.isfinite(f_lse)
                assert np.array_equal(fin, np.isfinite(c_lse))
                assert np.allclose(c_lse[fin], f_lse[fin], rtol=1e-6, atol=1e-6)
            # the gathered-row entry agrees with the full one
            Hc = H // W
            t, h = np.meshgrid(np.arange(T), np.arange(H), indexing="ij")
            t, h = t.ravel(), h.ravel()
            g_out, g_lse, _ = orc.fused_gathered(o[:, t, h], mx[:, t, h], sm[:, t, h], dt)
            j, hc = h // Hc, h % Hc
            assert np.array_equal(g_out, f_out[j, t, hc]) and np.array_equal(g_lse, f_lse[j, t, hc])


def pin_token_chain_equals_direct(orc):
    """The token-chunk exchange: pack(scatter_dim=0) -> all-to-all -> combine on
    the oracle's own packet equals the direct merge of every (t, h) in source
    order, exactly when every LSE is representable in float32 (sum = 1). This
    fixes where each combined row of the token-chunk variant lands: destination
    j holds tokens j*T/W .. (j+1)*T/W - 1 with all heads."""
    rng = np.random.default_rng(9)
    for W, T, H, D, dt in [(2, 4, 4, 8, BF16), (4, 8, 4, 16, FP16), (3, 6, 6, 8, BF16)]:
        o = rng.integers(0, 65535, size=(W, T, H, D), dtype=np.uint16)
        o = np.where((o & 0x7f80) == 0x7f80, o & 0x3fff, o).astype(np.uint16)
        if dt == FP16:
            o = np.where((o & 0x7c00) == 0x7c00, o & 0x3bff, o).astype(np.uint16)
        mx = rng.normal(0, 4, (W, T, H)).astype(np.float32)
        sm = np.ones((W, T, H), dtype=np.float32)
        sm[rng.random((W, T, H)) < 0.2] = 0.0
        sm[:, 1, 0] = 0.0                                   # one row invalid on every rank
        pkt, l32, _ = orc.pack(o, mx, sm, 0)                # [src][dst][T/W][H]
        c_out, c_lse, _ = orc.combine(orc.permute(pkt, W), orc.permute(l32, W), dt)
        d_out, d_lse, _ = orc.fused_gathered(o.reshape(W, T * H, D), mx.reshape(W, T * H),
                                             sm.reshape(W, T * H), dt)
        assert c_out.shape == (W, T // W, H, D)
        assert np.array_equal(c_out.reshape(T * H, D), d_out)
        assert np.array_equal(c_lse.reshape(T * H), d_lse)
        assert np.isneginf(c_lse.reshape(T, H)[1, 0]) and np.all(c_out.reshape(T, H, D)[1, 0] == 0)


ALL_PINS = [pin_lse_golden, pin_combine_golden, pin_bruteforce_attention, pin_combine_invariants,
            pin_payload_formats, pin_pack_layout, pin_pack_from_lse, pin_permute, pin_ulysses,
            pin_fused_equals_chain, pin_token_chain_equals_direct]
