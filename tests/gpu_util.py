"""Helpers for the GPU parity tests: moving generator/oracle arrays to and from
the device, and the tolerance checks the tests apply.

Tolerances (floating point):
  packet LSE   |lse_gpu - lse_ref| <= 2 ulp_f32(max(|lse_ref|, |max|, |ln sum|));
               -inf must match exactly, NaN never appears. ``ulp`` of the
               largest operand because m + ln s cancels: logf's own 1-ulp error
               is relative to ln s, not to the sum.
  combined LSE |dL| <= 2 ulp_f32(|L_ref| + ln W) + W * 2^-23 (+ the packet LSE
               bound of the contributions, for the fused path, where each LSE
               is formed on the fly).
  combined O   elementwise |o_gpu - o_ref| <= 1e-2 + 4e-3 |o_ref| (max abs
               1e-2 and relative 4e-3), every row with a nonzero reference
               ||o_gpu - o_ref||_2 <= 4e-3 ||o_ref||_2, all-invalid rows exactly
               +0, and -- tighter -- o_gpu within one payload ulp (+3e-5
               absolute, for fp32 accumulation near exact cancellation) of
               the nearest-even rounding of the float64 reference.
"""
from __future__ import annotations

import math

import numpy as np
import torch

BF16, FP16 = 0, 1
TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}
FMT = {"bf16": BF16, "fp16": FP16}


def dev_payload(bits: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TORCH_DT[dtype])
    return t.to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dev_f32(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def payload_values(bits: np.ndarray, dtype: str) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TORCH_DT[dtype])
    return t.double().numpy()


def ulp32(x) -> np.ndarray:
    x = np.abs(np.asarray(x, dtype=np.float64))
    x = np.minimum(x, 2.0 ** 127)
    return np.spacing(x.astype(np.float32)).astype(np.float64)


def safe_log(s: np.ndarray) -> np.ndarray:
    s = np.asarray(s, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(np.isfinite(s) & (s > 0), np.log(np.where(s > 0, s, 1.0)), 0.0)


def check_pack_lse(gpu: np.ndarray, ref: np.ndarray, m: np.ndarray, s: np.ndarray) -> None:
    """gpu float32, ref float64, m/s the statistics in the same layout."""
    gpu = np.asarray(gpu, dtype=np.float64)
    assert not np.isnan(gpu).any(), "NaN in the packet LSE"
    ninf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(gpu), ninf_ref), "invalid (-inf) pattern differs"
    fin = ~ninf_ref
    mag = np.maximum(np.abs(ref), np.maximum(np.abs(np.where(np.isfinite(m), m, 0)),
                                             np.abs(safe_log(s))))
    tol = 2 * ulp32(mag)
    with np.errstate(invalid="ignore"):
        err = np.abs(gpu - ref)
    bad = fin & (err > tol)
    assert not bad.any(), "LSE beyond 2 ulp at %d entries, e.g. gpu=%r ref=%r" % (
        bad.sum(), gpu[bad][:3], ref[bad][:3])


def lse_member_tol(m: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Per-row bound of the fused path's on-the-fly LSE error, m/s shaped [W, n]."""
    valid = np.isfinite(m) & np.isfinite(s) & (s > 0)
    lse = np.where(valid, m.astype(np.float64) + safe_log(s), 0.0)
    mag = np.maximum(np.abs(lse), np.maximum(np.abs(np.where(valid, m, 0)), np.abs(safe_log(s))))
    return np.where(valid, 2 * ulp32(mag), 0.0).max(axis=0)


def check_combined(out_bits: np.ndarray, out_lse: np.ndarray, ref: np.ndarray,
                   ref_lse: np.ndarray, ref_rounded: np.ndarray, dtype: str, W: int,
                   extra_lse_tol=0.0) -> None:
    """out_bits [..., D] payload bits, out_lse [...] float32 vs the float64 oracle."""
    D = out_bits.shape[-1]
    g = payload_values(out_bits, dtype).reshape(-1, D)
    r = np.asarray(ref, dtype=np.float64).reshape(-1, D)
    gl = np.asarray(out_lse, dtype=np.float64).reshape(-1)
    rl = np.asarray(ref_lse, dtype=np.float64).reshape(-1)
    extra = np.asarray(extra_lse_tol, dtype=np.float64)
    extra = np.broadcast_to(extra.reshape(-1) if extra.ndim else extra, rl.shape)
    # LSE
    assert not np.isnan(gl).any(), "NaN in the combined LSE"
    dead = np.isneginf(rl)
    assert np.array_equal(np.isneginf(gl), dead), "all-invalid rows differ"
    tol = 2 * ulp32(np.abs(rl) + math.log(max(W, 1))) + W * 2.0 ** -23 + extra
    with np.errstate(invalid="ignore"):
        err = np.abs(np.where(dead, 0, gl - rl))
    bad = err > tol
    assert not bad.any(), "combined LSE beyond tolerance at %d rows, max err %g (tol %g)" % (
        bad.sum(), err.max(), tol[np.argmax(err)])
    # all-invalid rows: exact +0
    if dead.any():
        assert np.all(out_bits.reshape(-1, D)[dead] == 0), "all-invalid rows are not +0"
    # O: max abs 1e-2 and relative 4e-3, elementwise
    diff = np.abs(g - r)
    bound = 1e-2 + 4e-3 * np.abs(r)
    assert np.all(diff <= bound), "O beyond 1e-2 + 4e-3|ref|: max excess %g" % (diff - bound).max()
    # row-relative L2
    nr = np.linalg.norm(r, axis=1)
    nd = np.linalg.norm(g - r, axis=1)
    rows = nr > 0
    if rows.any():
        rel = nd[rows] / nr[rows]
        assert rel.max() <= 4e-3, "row relative L2 error %g > 4e-3" % rel.max()
    # within one payload ulp of the correctly rounded reference
    rr = payload_values(ref_rounded, dtype).reshape(-1, D)
    ulp = np.spacing(np.abs(rr).astype(np.float16 if dtype == "fp16" else np.float32)).astype(
        np.float64)
    if dtype == "bf16":
        ulp = ulp * 2.0 ** 16   # float32 spacing -> bfloat16 spacing (16 fewer fraction bits)
        ulp = np.maximum(ulp, 2.0 ** -133)
    # fp32 accumulation can move a result across a rounding boundary (one ulp),
    # and near an exact cancellation its absolute error (~W 2^-24 max|o_r|)
    # exceeds the ulp of a near-zero result: allow 3e-5 absolute for that.
    excess = np.abs(g - rr) - (ulp * 1.0000001 + 3e-5)
    assert np.all(excess <= 0), "O more than one ulp from RNE(ref): max excess %g" % excess.max()
