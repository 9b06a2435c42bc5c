"""The seeded input generator: determinism, random access, distributions, patterns."""
import numpy as np
import torch

import synth


def test_deterministic_and_random_access():
    a = synth.fill(7, 3, synth.NORMAL, 0.0, 1.0, n=1000, start=500, fmt=synth.F64)
    b = synth.fill(7, 3, synth.NORMAL, 0.0, 1.0, n=1000, start=500, fmt=synth.F64)
    assert np.array_equal(a, b)
    idx = np.array([999 + 500, 500, 777, 501], dtype=np.uint64)
    c = synth.fill(7, 3, synth.NORMAL, 0.0, 1.0, idx=idx, fmt=synth.F64)
    assert np.array_equal(c, a[idx.astype(np.int64) - 500])
    assert not np.array_equal(a, synth.fill(8, 3, synth.NORMAL, 0.0, 1.0, n=1000, start=500, fmt=synth.F64))
    assert not np.array_equal(a, synth.fill(7, 4, synth.NORMAL, 0.0, 1.0, n=1000, start=500, fmt=synth.F64))


def _mix(z):
    M = 2**64 - 1
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
    return z ^ (z >> 31)


G = 0x9E3779B97F4A7C15
M64 = 2**64 - 1


def test_splitmix64_published_outputs():
    # SplitMix64 seeded with 0: the published first outputs of the generator
    assert [_mix((k * G) & M64) for k in (1, 2, 3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_c_draws_follow_the_stream_definition():
    # draw i of stream (seed, tid) = mix(state + (i + 1) * gamma),
    # state = mix(mix(seed + gamma) ^ (tid * 0xD1B54A32D192ED03 + 1))
    for seed, tid in [(0, 0), (1, 0x1000), (4, 0x9007)]:
        st = _mix(_mix((seed + G) & M64) ^ ((tid * 0xD1B54A32D192ED03 + 1) & M64))
        for i in (0, 1, 2, 12345, 2**40 + 7):
            assert synth.raw(seed, tid, i) == _mix((st + (i + 1) * G) & M64)


def test_distribution_moments():
    n = 400_000
    z = synth.fill(1, 1, synth.NORMAL, 2.0, 3.0, n=n, fmt=synth.F64)
    assert abs(z.mean() - 2.0) < 0.03 and abs(z.std() - 3.0) < 0.03
    assert abs(np.mean(np.abs((z - 2) / 3) < 1.0) - 0.6827) < 0.005
    u = synth.fill(1, 2, synth.UNIFORM, 1.0, 64.0, n=n, fmt=synth.F64)
    assert u.min() >= 1.0 and u.max() < 64.0 and abs(u.mean() - 32.5) < 0.2
    lu = synth.fill(1, 3, synth.LOGUNIFORM, 1e-3, 1e6, n=n, fmt=synth.F64)
    assert lu.min() >= 1e-3 and lu.max() <= 1e6
    ll = np.log10(lu)
    assert abs(ll.mean() - 1.5) < 0.05


def test_rounding_matches_libraries():
    x = synth.fill(5, 5, synth.NORMAL, 0.0, 1.0, n=20000, fmt=synth.F64) * 1000
    f16 = synth.fill(5, 5, synth.NORMAL, 0.0, 1.0, n=20000, fmt=synth.F16)
    assert np.array_equal(f16, (x / 1000).astype(np.float16).view(np.uint16))
    xf = synth.fill(5, 6, synth.NORMAL, 0.0, 1.0, n=20000, fmt=synth.F32)
    # float32 values: one rounding to bf16, torch as the reference
    bits = np.array([synth.round16(float(v), synth.BF16) for v in xf], dtype=np.uint16)
    want = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, want)


def test_workload_patterns():
    wl = synth.CONFIGS["tiny"]
    o, m, s = synth.full_inputs(wl)
    assert o.shape == (2, 64, 8, 64) and m.shape == (2, 64, 8)
    bad = ~np.isfinite(m) | ~np.isfinite(s) | ~(s > 0)
    assert 0.005 < bad.mean() < 0.05
    # rows and blocks agree
    t = np.array([0, 5, 63]); h = np.array([7, 0, 3])
    assert np.array_equal(synth.o_rows(wl, 1, t, h), o[1, t, h])
    mm, ss = synth.stats_at(wl, 1, t, h)
    assert np.array_equal(mm, m[1, t, h], equal_nan=True) and np.array_equal(ss, s[1, t, h])
    # mla: the last token is invalid on every rank and head
    mla = synth.CONFIGS["mla"]
    for r in (0, 7):
        mt, st = synth.stats_block(mla, r, mla.T - 2, mla.T)
        last_bad = ~np.isfinite(mt[1]) | ~np.isfinite(st[1]) | ~(st[1] > 0)
        assert last_bad.all()
    # stress: +/-inf maxima and zero sums near 1 %
    st = synth.CONFIGS["stress"]
    mt, sm = synth.stats_block(st, 3, 0, 512)
    assert 0.005 < np.isinf(mt).mean() < 0.02 and 0.005 < (sm == 0).mean() < 0.02
    assert (mt == np.inf).any() and (mt == -np.inf).any()
    # byte counts of the fused path
    assert synth.CONFIGS["decode"].fused_bytes() == 172_490_752
    assert synth.CONFIGS["tiny"].fused_bytes() == 206_848
