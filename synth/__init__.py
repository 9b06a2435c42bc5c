"""Seeded synthetic workloads for the DCP / Ulysses exchange path.

Both the CUDA path (through tests and the benchmark) and the CPU oracle take
their inputs from here. The module holds no part of the method's arithmetic:
it only draws numbers (``synth.c``) and places them in the tensor shapes and
invalid-statistic patterns that the workloads describe.

Workload shapes and distributions follow the five configurations of the
exchange benchmark: the vLLM-Ascend pull request "Fuse local SFA LSE formation
into DCP pack" (decode-context-parallel pack of partial outputs plus fp32
softmax max/sum, invalid-statistic cases in its test list) and the FastVideo
Ulysses all-to-all geometry (sequence-scatter / head-gather of bf16 q/k/v/o).
No public dataset is involved.

Element addressing: for rank ``r`` the partial output O_r[t][h][d] is element
``(t*H + h)*D + d`` of stream ``TID_O + r``; softmax_max / softmax_sum of
(t, h) are element ``t*H + h`` of their streams. Any element can be
regenerated independently, so full-size tensors never need to exist on the
host at once.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Tuple

import numpy as np

from . import build as _build

_lib = ctypes.CDLL(_build.build())
_lib.synth_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_double,
                            ctypes.c_double, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int64,
                            ctypes.c_int, ctypes.c_void_p]
_lib.synth_fill.restype = None
_lib.synth_raw.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
_lib.synth_raw.restype = ctypes.c_uint64
_lib.synth_round16.argtypes = [ctypes.c_double, ctypes.c_int]
_lib.synth_round16.restype = ctypes.c_uint16

NORMAL, UNIFORM, LOGUNIFORM, UNIT = 0, 1, 2, 3
F32, BF16, F16, F64 = 0, 1, 2, 3
_NP = {F32: np.float32, BF16: np.uint16, F16: np.uint16, F64: np.float64}

# stream ids (per-rank streams add the rank)
TID_O = 0x1000
TID_MAX = 0x2000
TID_SUM = 0x3000
TID_BAD = 0x4000        # per-entry invalid mask
TID_KIND = 0x5000       # which invalid kind
TID_BADTOK = 0x6000     # whole-token invalid mask (index t)
TID_MAXINF = 0x7000     # stress: max set to +/-inf
TID_MAXSIGN = 0x8000    # stress: sign of that inf
TID_SUMZERO = 0x9000    # stress: sum set to 0
TID_SEQ = 0xA000        # Ulysses sequence-sharded q/k/v
TID_HEAD = 0xB000       # Ulysses head-sharded o
TID_LSE = 0xC000        # direct LSE inputs for the combine-only cases


def fill(seed: int, tid: int, dist: int, p0: float, p1: float, n: int = 0, start: int = 0,
         idx: Optional[np.ndarray] = None, fmt: int = F32,
         out: Optional[np.ndarray] = None) -> np.ndarray:
    """Draw n values (or one per entry of ``idx``) from stream (seed, tid), into
    ``out`` (a C-contiguous array of n elements of the format's type) if given."""
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.uint64)
        n = idx.size
    if out is None:
        out = np.empty(n, dtype=_NP[fmt])
    else:
        if out.dtype != _NP[fmt] or out.size != n or not out.flags.c_contiguous:
            raise ValueError("out must be C-contiguous %s with %d elements" % (_NP[fmt], n))
        out = out.reshape(-1)
    if n:
        _lib.synth_fill(seed, tid, dist, p0, p1, start,
                        idx.ctypes.data if idx is not None else None, n, fmt, out.ctypes.data)
    return out


def raw(seed: int, tid: int, i: int) -> int:
    return int(_lib.synth_raw(seed, tid, i))


def round16(x: float, fmt: int) -> int:
    return int(_lib.synth_round16(x, fmt))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One exchange workload: W simulated ranks, T tokens, H heads, head dim D."""
    name: str
    W: int
    T: int
    H: int
    D: int
    dtype: str = "bf16"                  # payload dtype: "bf16" or "fp16"
    seed: int = 0
    o_sigma: float = 1.0                 # O ~ N(0, o_sigma)
    max_sigma: float = 1.0               # softmax_max ~ N(0, max_sigma)
    sum_dist: Tuple[int, float, float] = (UNIFORM, 1.0, 64.0)
    p_invalid: float = 0.0               # per-entry: NaN max / +inf sum / sum = 0
    p_token_invalid: float = 0.0         # whole token invalid on every (r, h)
    last_token_invalid: bool = False
    p_max_inf: float = 0.0               # max = +/-inf (sign 50/50)
    p_sum_zero: float = 0.0              # sum = 0 (independent of the above)
    ulysses_B: Tuple[int, int] = (3, 1)  # batch planes of the seq->head and head->seq operands

    @property
    def Hc(self) -> int:
        return self.H // self.W

    @property
    def fmt(self) -> int:
        return BF16 if self.dtype == "bf16" else F16

    @property
    def e(self) -> int:
        return 2

    def fused_bytes(self) -> int:
        """Algorithmic HBM bytes of one fused pack->permute->combine call."""
        rows = self.T * self.H
        return self.W * rows * (self.D * self.e + 8) + rows * (self.D * self.e + 4)

    def pack_bytes(self) -> int:
        rows = self.T * self.H
        return self.W * rows * (2 * self.D * self.e + 12)

    def permute_bytes(self) -> int:
        rows = self.T * self.H
        return 2 * self.W * rows * (self.D * self.e + 4)

    def combine_bytes(self) -> int:
        rows = self.T * self.H
        return (self.W + 1) * rows * (self.D * self.e + 4)


CONFIGS = {
    "tiny": Workload("tiny", W=2, T=64, H=8, D=64, dtype="bf16", seed=0, o_sigma=1.0,
                     max_sigma=3.0, sum_dist=(UNIFORM, 1.0, 64.0), p_invalid=0.02),
    "decode": Workload("decode", W=4, T=4096, H=32, D=128, dtype="bf16", seed=1, o_sigma=1.0,
                       max_sigma=5.0, sum_dist=(UNIFORM, 1.0, 4096.0), p_invalid=0.005),
    "mla": Workload("mla", W=8, T=8192, H=128, D=512, dtype="bf16", seed=2, o_sigma=0.5,
                    max_sigma=8.0, sum_dist=(LOGUNIFORM, 1.0, 1e5), p_invalid=0.01,
                    p_token_invalid=0.001, last_token_invalid=True),
    "ulysses": Workload("ulysses", W=8, T=32768, H=48, D=128, dtype="bf16", seed=3, o_sigma=1.0,
                        max_sigma=4.0, sum_dist=(UNIFORM, 1.0, 8192.0)),
    "stress": Workload("stress", W=16, T=65536, H=64, D=128, dtype="fp16", seed=4, o_sigma=2.0,
                       max_sigma=10.0, sum_dist=(LOGUNIFORM, 1e-3, 1e6), p_max_inf=0.01,
                       p_sum_zero=0.01),
}


# ----------------------------------------------------------------------------------------------
# partial outputs O_r[t][h][:]

def o_block(wl: Workload, r: int, t0: int = 0, t1: Optional[int] = None,
            out: Optional[np.ndarray] = None) -> np.ndarray:
    """O_r[t0:t1] as raw 16-bit payload, shape [t1-t0, H, D] (written into
    ``out``, a C-contiguous uint16 array of that size, if given)."""
    t1 = wl.T if t1 is None else t1
    n = (t1 - t0) * wl.H * wl.D
    v = fill(wl.seed, TID_O + r, NORMAL, 0.0, wl.o_sigma, n=n, start=t0 * wl.H * wl.D, fmt=wl.fmt,
             out=out)
    return v.reshape(t1 - t0, wl.H, wl.D)


def o_rows(wl: Workload, r: int, t: np.ndarray, h: np.ndarray) -> np.ndarray:
    """Rows O_r[t[k]][h[k]][:] as raw 16-bit payload, shape [len(t), D]."""
    t = np.asarray(t, dtype=np.uint64)
    h = np.asarray(h, dtype=np.uint64)
    base = (t * np.uint64(wl.H) + h) * np.uint64(wl.D)
    idx = (base[:, None] + np.arange(wl.D, dtype=np.uint64)[None, :]).reshape(-1)
    v = fill(wl.seed, TID_O + r, NORMAL, 0.0, wl.o_sigma, idx=idx, fmt=wl.fmt)
    return v.reshape(t.size, wl.D)


# ----------------------------------------------------------------------------------------------
# softmax statistics with the workload's invalid pattern

def _stats(wl: Workload, r: int, flat: np.ndarray, t: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    m = fill(wl.seed, TID_MAX + r, NORMAL, 0.0, wl.max_sigma, idx=flat, fmt=F32)
    dist, a, b = wl.sum_dist
    s = fill(wl.seed, TID_SUM + r, dist, a, b, idx=flat, fmt=F32)
    bad = np.zeros(flat.size, dtype=bool)
    if wl.p_invalid > 0:
        bad |= fill(wl.seed, TID_BAD + r, UNIT, 0, 0, idx=flat, fmt=F64) < wl.p_invalid
    if wl.p_token_invalid > 0 or wl.last_token_invalid:
        badtok = fill(wl.seed, TID_BADTOK, UNIT, 0, 0, idx=t, fmt=F64) < wl.p_token_invalid
        if wl.last_token_invalid:
            badtok |= t == wl.T - 1
        bad |= badtok
    if bad.any():
        kind = np.floor(fill(wl.seed, TID_KIND + r, UNIT, 0, 0, idx=flat, fmt=F64) * 3).astype(np.int64)
        m = np.where(bad & (kind == 0), np.float32(np.nan), m)
        s = np.where(bad & (kind == 1), np.float32(np.inf), s)
        s = np.where(bad & (kind == 2), np.float32(0.0), s)
    if wl.p_max_inf > 0:
        hit = fill(wl.seed, TID_MAXINF + r, UNIT, 0, 0, idx=flat, fmt=F64) < wl.p_max_inf
        pos = fill(wl.seed, TID_MAXSIGN + r, UNIT, 0, 0, idx=flat, fmt=F64) < 0.5
        m = np.where(hit, np.where(pos, np.float32(np.inf), np.float32(-np.inf)), m)
    if wl.p_sum_zero > 0:
        hit = fill(wl.seed, TID_SUMZERO + r, UNIT, 0, 0, idx=flat, fmt=F64) < wl.p_sum_zero
        s = np.where(hit, np.float32(0.0), s)
    return m.astype(np.float32), s.astype(np.float32)


def stats_block(wl: Workload, r: int, t0: int = 0, t1: Optional[int] = None):
    """(softmax_max, softmax_sum) of rank r for tokens t0:t1, each float32 [t1-t0, H]."""
    t1 = wl.T if t1 is None else t1
    t = np.repeat(np.arange(t0, t1, dtype=np.uint64), wl.H)
    flat = np.arange(t0 * wl.H, t1 * wl.H, dtype=np.uint64)
    m, s = _stats(wl, r, flat, t)
    return m.reshape(t1 - t0, wl.H), s.reshape(t1 - t0, wl.H)


def stats_at(wl: Workload, r: int, t: np.ndarray, h: np.ndarray):
    t = np.asarray(t, dtype=np.uint64)
    h = np.asarray(h, dtype=np.uint64)
    return _stats(wl, r, t * np.uint64(wl.H) + h, t)


def full_inputs(wl: Workload):
    """All inputs at once (small workloads only): O [W,T,H,D] u16, max and sum [W,T,H] f32."""
    o = np.stack([o_block(wl, r) for r in range(wl.W)])
    ms = [stats_block(wl, r) for r in range(wl.W)]
    return o, np.stack([a for a, _ in ms]), np.stack([b for _, b in ms])


# ----------------------------------------------------------------------------------------------
# direct inputs for the combine-only entry point (received packet)

def received_lse(wl: Workload, p_neg_inf: float, n: int, sigma: float = 6.0) -> np.ndarray:
    """[W, n] float32 LSE values ~ N(0, sigma) with a fraction set to -inf, one stream per rank."""
    rows = []
    for r in range(wl.W):
        v = fill(wl.seed, TID_LSE + r, NORMAL, 0.0, sigma, n=n, fmt=F32)
        dead = fill(wl.seed, TID_LSE + 0x100 + r, UNIT, 0, 0, n=n, fmt=F64) < p_neg_inf
        rows.append(np.where(dead, np.float32(-np.inf), v).astype(np.float32))
    return np.stack(rows)


# ----------------------------------------------------------------------------------------------
# Ulysses operands

def ulysses_seq_block(wl: Workload, r: int) -> np.ndarray:
    """Rank r's sequence shard [B, S/W, H, D] (bf16 bits) for the seq->head transform."""
    B = wl.ulysses_B[0]
    S_l = wl.T // wl.W
    n = B * S_l * wl.H * wl.D
    return fill(wl.seed, TID_SEQ + r, NORMAL, 0.0, wl.o_sigma, n=n, fmt=wl.fmt).reshape(
        B, S_l, wl.H, wl.D)


def ulysses_head_block(wl: Workload, r: int) -> np.ndarray:
    """Rank r's head shard [B, S, H/W, D] (bf16 bits) for the head->seq transform."""
    B = wl.ulysses_B[1]
    n = B * wl.T * wl.Hc * wl.D
    return fill(wl.seed, TID_HEAD + r, NORMAL, 0.0, wl.o_sigma, n=n, fmt=wl.fmt).reshape(
        B, wl.T, wl.Hc, wl.D)


def threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
