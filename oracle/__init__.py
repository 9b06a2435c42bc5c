"""CPU oracle for the DCP exchange (pack -> all-to-all -> stable combine) and the
Ulysses layout transforms: plain float64 loops in ``cplse_oracle.c``.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package. The CUDA
library never calls it and shares no code with it.

Arrays are numpy: payloads are raw 16-bit patterns (``np.uint16``) of bf16 or
fp16, statistics are ``np.float32``, results are ``np.float64`` (plus an
optional nearest-even rounding back to the payload format).
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import build as _build

BF16, FP16 = 0, 1

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _check_split(W: int, T: int, H: int, scatter_dim: int) -> None:
    """The packet splits heads (and, for token chunks, tokens) evenly over W ranks."""
    assert W >= 1 and H % W == 0, "H = %d must be a multiple of W = %d" % (H, W)
    assert scatter_dim in (0, 1) and (scatter_dim == 1 or T % W == 0), \
        "token chunks need T %% W == 0 (T = %d, W = %d)" % (T, W)


def _elem_strides(a: np.ndarray):
    return [s // a.itemsize for s in a.strides]


class Oracle:
    """ctypes view of one build of the oracle library (the tests also load mutants)."""

    def __init__(self, path: Optional[str] = None):
        self.lib = lib = ctypes.CDLL(path or _build.build())
        lib.oracle_lse.argtypes = [ctypes.c_double, ctypes.c_double]
        lib.oracle_lse.restype = ctypes.c_double
        lib.oracle_payload_value.argtypes = [ctypes.c_uint16, ctypes.c_int]
        lib.oracle_payload_value.restype = ctypes.c_double
        lib.oracle_payload_round.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.oracle_payload_round.restype = ctypes.c_uint16
        lib.oracle_pack.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _i64, _i64, _p, _i64, _i64,
                                    _i64, ctypes.c_int, _i64, _i64, _i64, ctypes.c_int, _p, _p, _p]
        lib.oracle_pack_from_lse.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _i64, _i64,
                                             ctypes.c_int, _i64, _i64, _i64, ctypes.c_int, _p, _p]
        lib.oracle_permute.argtypes = [_p, _p, ctypes.c_int, _i64]
        lib.oracle_combine_f64.argtypes = [ctypes.c_int, _i64, _i64, _p, _p, _p, _p]
        lib.oracle_combine.argtypes = [_p, _p, ctypes.c_int, _i64, _i64, ctypes.c_int, _p, _p, _p]
        lib.oracle_fused.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _i64, _i64, _p, _i64, _i64,
                                     _i64, ctypes.c_int, _i64, _i64, _i64, ctypes.c_int, _p, _p,
                                     _p]
        lib.oracle_fused_gathered.argtypes = [_p, _p, _p, ctypes.c_int, _i64, _i64, ctypes.c_int,
                                              _p, _p, _p]
        for f in ("oracle_seq2head", "oracle_head2seq"):
            getattr(lib, f).argtypes = [_p, _p, ctypes.c_int, _i64, _i64, _i64, _i64, _i64]
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = ctypes.c_int
        for f in ("oracle_pack", "oracle_pack_from_lse", "oracle_permute", "oracle_combine_f64", "oracle_combine",
                  "oracle_fused", "oracle_fused_gathered", "oracle_seq2head", "oracle_head2seq"):
            getattr(lib, f).restype = None

    # -- threads of the parallel loops ---------------------------------------------------------
    def threads(self) -> int:
        return int(self.lib.oracle_threads())

    def set_threads(self, n: int) -> int:
        return int(self.lib.oracle_set_threads(int(n)))

    # -- scalar helpers ----------------------------------------------------------------------
    def lse(self, m: float, s: float) -> float:
        return self.lib.oracle_lse(float(m), float(s))

    def payload_value(self, bits: int, dtype: int) -> float:
        return self.lib.oracle_payload_value(int(bits), dtype)

    def payload_round(self, x: float, dtype: int) -> int:
        return int(self.lib.oracle_payload_round(float(x), dtype))

    # -- pack --------------------------------------------------------------------------------
    def pack(self, o: np.ndarray, mx: np.ndarray, sm: np.ndarray, scatter_dim: int = 1):
        """o [W,T,H,D] u16 (any strides, D contiguous), max/sum [W,T,H] f32 ->
        (pkt_o u16, pkt_lse32 f32, pkt_lse64 f64), destination-major packet."""
        W, T, H, D = o.shape
        assert o.dtype == np.uint16 and o.strides[3] == 2
        assert mx.dtype == np.float32 and sm.dtype == np.float32
        _check_split(W, T, H, scatter_dim)
        if scatter_dim == 1:
            shape = (W, W, T, H // W)
        else:
            shape = (W, W, T // W, H)
        pkt_o = np.empty(shape + (D,), dtype=np.uint16)
        l32 = np.empty(shape, dtype=np.float32)
        l64 = np.empty(shape, dtype=np.float64)
        self.lib.oracle_pack(o.ctypes.data, *_elem_strides(o)[:3], mx.ctypes.data,
                             *_elem_strides(mx), sm.ctypes.data, *_elem_strides(sm), W, T, H, D,
                             scatter_dim, pkt_o.ctypes.data, l32.ctypes.data, l64.ctypes.data)
        return pkt_o, l32, l64

    def materialize_lse(self, mx: np.ndarray, sm: np.ndarray) -> np.ndarray:
        """The legacy first step, element by element: float64 LSE of max/sum arrays."""
        return np.vectorize(self.lse, otypes=[np.float64])(mx.astype(np.float64),
                                                           sm.astype(np.float64))

    def pack_from_lse(self, o: np.ndarray, lse: np.ndarray, scatter_dim: int = 1):
        """o [W,T,H,D] u16, lse [W,T,H] f32 (any strides) -> (pkt_o, pkt_lse), legacy pack."""
        W, T, H, D = o.shape
        assert o.dtype == np.uint16 and o.strides[3] == 2 and lse.dtype == np.float32
        _check_split(W, T, H, scatter_dim)
        shape = (W, W, T, H // W) if scatter_dim == 1 else (W, W, T // W, H)
        pkt_o = np.empty(shape + (D,), dtype=np.uint16)
        pkt_l = np.empty(shape, dtype=np.float32)
        self.lib.oracle_pack_from_lse(o.ctypes.data, *_elem_strides(o)[:3], lse.ctypes.data,
                                      *_elem_strides(lse), W, T, H, D, scatter_dim,
                                      pkt_o.ctypes.data, pkt_l.ctypes.data)
        return pkt_o, pkt_l

    # -- all-to-all permutation --------------------------------------------------------------
    def permute(self, send: np.ndarray, W: int) -> np.ndarray:
        """send viewed as W*W equal blocks [src][dst] -> recv [dst][src], same shape."""
        send = np.ascontiguousarray(send)
        assert send.nbytes % (W * W) == 0
        recv = np.empty_like(send)
        self.lib.oracle_permute(send.ctypes.data, recv.ctypes.data, W, send.nbytes // (W * W))
        return recv

    # -- combine -----------------------------------------------------------------------------
    def combine_f64(self, o: np.ndarray, lse: np.ndarray):
        """o [W,N,D] f64, lse [W,N] f64 -> out [N,D], out_lse [N]."""
        o = np.ascontiguousarray(o, dtype=np.float64)
        lse = np.ascontiguousarray(lse, dtype=np.float64)
        W, N, D = o.shape
        out = np.empty((N, D))
        out_lse = np.empty(N)
        self.lib.oracle_combine_f64(W, N, D, o.ctypes.data, lse.ctypes.data, out.ctypes.data,
                                    out_lse.ctypes.data)
        return out, out_lse

    def combine(self, recv_o: np.ndarray, recv_lse: np.ndarray, dtype: int):
        """recv_o [W_dst,W_src,*rows,D] u16, recv_lse [W_dst,W_src,*rows] f32 ->
        (out f64 [W_dst,*rows,D], out_lse f64 [W_dst,*rows], out_rounded u16)."""
        recv_o = np.ascontiguousarray(recv_o)
        recv_lse = np.ascontiguousarray(recv_lse, dtype=np.float32)
        W = recv_o.shape[0]
        D = recv_o.shape[-1]
        rows = recv_o.shape[2:-1]
        N = int(np.prod(rows)) if rows else 1
        out = np.empty((W,) + rows + (D,))
        out_lse = np.empty((W,) + rows)
        rounded = np.empty((W,) + rows + (D,), dtype=np.uint16)
        self.lib.oracle_combine(recv_o.ctypes.data, recv_lse.ctypes.data, W, N, D, dtype,
                                out.ctypes.data, out_lse.ctypes.data, rounded.ctypes.data)
        return out, out_lse, rounded

    # -- fused -------------------------------------------------------------------------------
    def fused(self, o: np.ndarray, mx: np.ndarray, sm: np.ndarray, dtype: int):
        """o [W,T,H,D] u16, max/sum [W,T,H] f32 -> (out [W,T,Hc,D] f64, out_lse [W,T,Hc], rounded)."""
        W, T, H, D = o.shape
        assert o.strides[3] == 2
        _check_split(W, T, H, 1)
        out = np.empty((W, T, H // W, D))
        out_lse = np.empty((W, T, H // W))
        rounded = np.empty((W, T, H // W, D), dtype=np.uint16)
        self.lib.oracle_fused(o.ctypes.data, *_elem_strides(o)[:3], mx.ctypes.data,
                              *_elem_strides(mx), sm.ctypes.data, *_elem_strides(sm), W, T, H, D,
                              dtype, out.ctypes.data, out_lse.ctypes.data, rounded.ctypes.data)
        return out, out_lse, rounded

    def fused_gathered(self, o: np.ndarray, mx: np.ndarray, sm: np.ndarray, dtype: int):
        """o [W,n,D] u16, max/sum [W,n] f32 -> (out [n,D] f64, out_lse [n], rounded)."""
        o = np.ascontiguousarray(o, dtype=np.uint16)
        mx = np.ascontiguousarray(mx, dtype=np.float32)
        sm = np.ascontiguousarray(sm, dtype=np.float32)
        W, n, D = o.shape
        out = np.empty((n, D))
        out_lse = np.empty(n)
        rounded = np.empty((n, D), dtype=np.uint16)
        self.lib.oracle_fused_gathered(o.ctypes.data, mx.ctypes.data, sm.ctypes.data, W, n, D,
                                       dtype, out.ctypes.data, out_lse.ctypes.data,
                                       rounded.ctypes.data)
        return out, out_lse, rounded

    # -- Ulysses -----------------------------------------------------------------------------
    def seq2head(self, x: np.ndarray) -> np.ndarray:
        """x [W,B,S_l,H,D] -> [W,B,S,H/W,D] (any 1/2/4-byte element type)."""
        x = np.ascontiguousarray(x)
        W, B, S_l, H, D = x.shape
        out = np.empty((W, B, S_l * W, H // W, D), dtype=x.dtype)
        self.lib.oracle_seq2head(x.ctypes.data, out.ctypes.data, W, B, S_l, H, D, x.itemsize)
        return out

    def head2seq(self, x: np.ndarray) -> np.ndarray:
        """x [W,B,S,Hc,D] -> [W,B,S/W,Hc*W,D]."""
        x = np.ascontiguousarray(x)
        W, B, S, Hc, D = x.shape
        out = np.empty((W, B, S // W, Hc * W, D), dtype=x.dtype)
        self.lib.oracle_head2seq(x.ctypes.data, out.ctypes.data, W, B, S // W, Hc * W, D,
                                 x.itemsize)
        return out


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
