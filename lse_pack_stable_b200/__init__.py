"""Python binding of libcplse (include/cplse.h): argument marshalling only.

Every function has the name of its C entry point, takes torch CUDA tensors,
passes their device pointers, sizes and strides through the C-ABI, and
enqueues the work on the current torch stream (or ``stream=``). Outputs are
allocated with ``torch.empty`` when not given. Nothing here computes any part
of the method: there is no fallback path. If the shared library is missing or
a call fails, a ``RuntimeError`` carries the library's message.

Layouts (W ranks, T tokens, H heads, Hc = H/W, D head dim):
    o            [W, T, H, D]   bf16/fp16, D contiguous, other strides free
    smax, ssum   [W, T, H]      float32, any strides
    pkt_o        [W, W, T, Hc, D] (heads) or [W, W, T/W, H, D] (tokens)
    pkt_lse      [W, W, T, Hc]    or [W, W, T/W, H]   float32
    out          [W, T, Hc, D],  out_lse [W, T, Hc]
    Ulysses      [W, B, S/W, H, D] <-> [W, B, S, Hc, D]
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libcplse.so")

if not os.path.exists(LIBRARY_PATH):
    raise ImportError("libcplse.so is not built: run `python lse_pack_stable_b200/build.py` "
                      "(or __graft_entry__.build())")

_lib = ctypes.CDLL(LIBRARY_PATH)

CP_OK, CP_ERR_ARG, CP_ERR_SHAPE, CP_ERR_ALIGN, CP_ERR_ALIAS, CP_ERR_UNSUPPORTED, CP_ERR_CUDA = (
    0, -1, -2, -3, -4, -5, -6)
CP_BF16, CP_FP16 = 0, 1
STATUS_NAMES = {0: "CP_OK", -1: "CP_ERR_ARG", -2: "CP_ERR_SHAPE", -3: "CP_ERR_ALIGN",
                -4: "CP_ERR_ALIAS", -5: "CP_ERR_UNSUPPORTED", -6: "CP_ERR_CUDA"}
EXPORTS = ("cp_abi_version", "cp_last_error", "cp_pack_lse", "cp_lse_materialize",
           "cp_pack_from_lse", "cp_a2a_local_permute",
           "cp_lse_combine", "cp_pack_permute_combine_fused", "cp_pack_lse_rank",
           "cp_lse_combine_rank", "cp_pull_combine", "cp_ipc_export", "cp_ipc_import",
           "cp_ipc_close", "ulysses_seq2head", "ulysses_head2seq", "ulysses_seq2head_pull",
           "ulysses_head2seq_pull")


class Strides3(ctypes.Structure):
    _fields_ = [("r", ctypes.c_int64), ("t", ctypes.c_int64), ("h", ctypes.c_int64)]


_p, _i, _i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
_lib.cp_abi_version.argtypes = []
_lib.cp_abi_version.restype = _i
ABI_VERSION = 4           # include/cplse.h CPLSE_ABI_VERSION this binding marshals for
if _lib.cp_abi_version() != ABI_VERSION:
    raise ImportError("libcplse.so has ABI version %d, this binding needs %d: rebuild it with "
                      "`python lse_pack_stable_b200/build.py`" % (_lib.cp_abi_version(), ABI_VERSION))
_lib.cp_last_error.argtypes = []
_lib.cp_last_error.restype = ctypes.c_char_p
_lib.cp_pack_lse.argtypes = [_p, Strides3, _p, Strides3, _p, Strides3, _i, _i64, _i, _i, _i, _i,
                             _p, _p, _p]
_lib.cp_lse_materialize.argtypes = [_p, Strides3, _p, Strides3, _i, _i64, _i, _p, _p]
_lib.cp_pack_from_lse.argtypes = [_p, Strides3, _p, Strides3, _i, _i64, _i, _i, _i, _i, _p, _p, _p]
_lib.cp_a2a_local_permute.argtypes = [_p, _p, _i, _i64, _p]
_lib.cp_lse_combine.argtypes = [_p, _p, _i, _i64, _i, _i, _i, _p, _p, _p]
_lib.cp_pack_permute_combine_fused.argtypes = [_p, Strides3, _p, Strides3, _p, Strides3, _i, _i64,
                                               _i, _i, _i, _i, _p, _p, _p]
_lib.cp_pack_lse_rank.argtypes = [_p, Strides3, _p, Strides3, _p, Strides3, _i, _i64, _i, _i, _i,
                                  _i, _p, _p, _p]
_lib.cp_lse_combine_rank.argtypes = [_p, _p, _i, _i64, _i, _i, _i, _p, _p, _p]
_lib.cp_pull_combine.argtypes = [_p, Strides3, _p, Strides3, _p, Strides3, _i, _i64, _i, _i, _i,
                                 _i, _i, _p, _p, _p]


class IpcHandle(ctypes.Structure):
    """cp_ipc_handle of include/cplse.h."""
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_int64),
                ("alloc_bytes", ctypes.c_int64), ("device", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_lib.cp_ipc_export.argtypes = [_p, ctypes.POINTER(IpcHandle)]
_lib.cp_ipc_import.argtypes = [ctypes.POINTER(IpcHandle), ctypes.POINTER(ctypes.c_void_p),
                               ctypes.POINTER(ctypes.c_void_p)]
_lib.cp_ipc_close.argtypes = [_p]
_lib.ulysses_seq2head.argtypes = [_p, _p, _i, _i, _i64, _i, _i, _i, _p]
_lib.ulysses_head2seq.argtypes = [_p, _p, _i, _i, _i64, _i, _i, _i, _p]
_lib.ulysses_seq2head_pull.argtypes = [_p, _p, _i, _i, _i64, _i, _i, _i, _i, _p]
_lib.ulysses_head2seq_pull.argtypes = [_p, _p, _i, _i, _i64, _i, _i, _i, _i, _p]
for _f in ("cp_pack_lse", "cp_lse_materialize", "cp_pack_from_lse", "cp_a2a_local_permute",
           "cp_lse_combine", "cp_pack_permute_combine_fused", "cp_pack_lse_rank",
           "cp_lse_combine_rank", "cp_pull_combine", "cp_ipc_export", "cp_ipc_import",
           "cp_ipc_close", "ulysses_seq2head", "ulysses_head2seq", "ulysses_seq2head_pull",
           "ulysses_head2seq_pull"):
    getattr(_lib, _f).restype = _i


class CplseError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), message))
        self.status = status


def _check(status: int) -> None:
    if status != CP_OK:
        raise CplseError(status, _lib.cp_last_error().decode())


def _dtype(t) -> int:
    if t.dtype == torch.bfloat16:
        return CP_BF16
    if t.dtype == torch.float16:
        return CP_FP16
    raise TypeError("payload dtype must be bfloat16 or float16, got %s" % t.dtype)


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _strides3(t: torch.Tensor) -> Strides3:
    st = t.stride()
    if t.dim() == 4 and st[3] != 1:
        raise ValueError("the head dim (last) of o must be contiguous")
    return Strides3(st[0], st[1], st[2])


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dense(t: torch.Tensor, name: str) -> None:
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _expect(t: torch.Tensor, name: str, shape, dtype, device: torch.device) -> None:
    """The C layer derives every extent from the sizes it is given, so a tensor
    of another shape, type or device would be read or written out of bounds:
    refuse it here."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))


def _payload(t: torch.Tensor, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dim() != ndim:
        raise ValueError("%s must have %d dimensions, got shape %s" % (name, ndim, tuple(t.shape)))
    _dtype(t)


def _stats(o: torch.Tensor, smax: torch.Tensor, ssum: torch.Tensor) -> None:
    W, T, H = o.shape[:3]
    _expect(smax, "smax", (W, T, H), torch.float32, o.device)
    _expect(ssum, "ssum", (W, T, H), torch.float32, o.device)


def _split(n: int, W: int, what: str) -> int:
    if W < 1 or n % W != 0:
        raise ValueError("%s = %d is not a multiple of W = %d" % (what, n, W))
    return n // W


def abi_version() -> int:
    return _lib.cp_abi_version()


def last_error() -> str:
    return _lib.cp_last_error().decode()


def _packet_shape(W: int, T: int, H: int, scatter_dim: int):
    if scatter_dim == 1:
        return (W, W, T, _split(H, W, "H"))
    if scatter_dim == 0:
        return (W, W, _split(T, W, "T"), H)
    raise ValueError("scatter_dim must be 0 (tokens) or 1 (heads), got %r" % (scatter_dim,))


def cp_pack_lse(o: torch.Tensor, smax: torch.Tensor, ssum: torch.Tensor, scatter_dim: int = 1,
                pkt_o: Optional[torch.Tensor] = None, pkt_lse: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    _payload(o, "o", 4)
    W, T, H, D = o.shape
    _stats(o, smax, ssum)
    shape = _packet_shape(W, T, H, scatter_dim)
    if pkt_o is None:
        pkt_o = torch.empty(shape + (D,), dtype=o.dtype, device=o.device)
    if pkt_lse is None:
        pkt_lse = torch.empty(shape, dtype=torch.float32, device=o.device)
    _expect(pkt_o, "pkt_o", shape + (D,), o.dtype, o.device)
    _expect(pkt_lse, "pkt_lse", shape, torch.float32, o.device)
    _dense(pkt_o, "pkt_o")
    _dense(pkt_lse, "pkt_lse")
    _check(_lib.cp_pack_lse(_ptr(o), _strides3(o), _ptr(smax), _strides3(smax), _ptr(ssum),
                            _strides3(ssum), W, T, H, D, _dtype(o), scatter_dim, _ptr(pkt_o),
                            _ptr(pkt_lse), _stream(stream)))
    return pkt_o, pkt_lse


def cp_lse_materialize(smax: torch.Tensor, ssum: torch.Tensor, lse: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """Legacy first step: LSE [W, T, H] float32 from softmax max/sum."""
    if not isinstance(smax, torch.Tensor) or smax.dim() != 3:
        raise ValueError("smax must be a [W, T, H] tensor")
    W, T, H = smax.shape
    _expect(smax, "smax", (W, T, H), torch.float32, smax.device)
    _expect(ssum, "ssum", (W, T, H), torch.float32, smax.device)
    if lse is None:
        lse = torch.empty((W, T, H), dtype=torch.float32, device=smax.device)
    _expect(lse, "lse", (W, T, H), torch.float32, smax.device)
    _dense(lse, "lse")
    _check(_lib.cp_lse_materialize(_ptr(smax), _strides3(smax), _ptr(ssum), _strides3(ssum), W, T,
                                   H, _ptr(lse), _stream(stream)))
    return lse


def cp_pack_from_lse(o: torch.Tensor, lse: torch.Tensor, scatter_dim: int = 1,
                     pkt_o: Optional[torch.Tensor] = None, pkt_lse: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Legacy pack: the packet of cp_pack_lse, its LSE region copied from `lse`."""
    _payload(o, "o", 4)
    W, T, H, D = o.shape
    _expect(lse, "lse", (W, T, H), torch.float32, o.device)
    shape = _packet_shape(W, T, H, scatter_dim)
    if pkt_o is None:
        pkt_o = torch.empty(shape + (D,), dtype=o.dtype, device=o.device)
    if pkt_lse is None:
        pkt_lse = torch.empty(shape, dtype=torch.float32, device=o.device)
    _expect(pkt_o, "pkt_o", shape + (D,), o.dtype, o.device)
    _expect(pkt_lse, "pkt_lse", shape, torch.float32, o.device)
    _dense(pkt_o, "pkt_o")
    _dense(pkt_lse, "pkt_lse")
    _check(_lib.cp_pack_from_lse(_ptr(o), _strides3(o), _ptr(lse), _strides3(lse), W, T, H, D,
                                 _dtype(o), scatter_dim, _ptr(pkt_o), _ptr(pkt_lse),
                                 _stream(stream)))
    return pkt_o, pkt_lse


def cp_a2a_local_permute(send: torch.Tensor, W: int, recv: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """send: any contiguous tensor whose bytes are W*W equal blocks [src][dst]."""
    if recv is None:
        recv = torch.empty_like(send)
    _dense(send, "send")
    _dense(recv, "recv")
    nbytes = send.numel() * send.element_size()
    if recv.numel() * recv.element_size() != nbytes or recv.device != send.device:
        raise ValueError("recv must have the bytes (%d) and device (%s) of send"
                         % (nbytes, send.device))
    if nbytes % (W * W) != 0:
        raise ValueError("send bytes (%d) are not W*W equal blocks" % nbytes)
    _check(_lib.cp_a2a_local_permute(_ptr(send), _ptr(recv), W, nbytes // (W * W),
                                     _stream(stream)))
    return recv


def cp_lse_combine(recv_o: torch.Tensor, recv_lse: torch.Tensor,
                   out: Optional[torch.Tensor] = None, out_lse: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """recv_o [W, W, T, Hc, D], recv_lse [W, W, T, Hc] -> out [W, T, Hc, D], out_lse [W, T, Hc]."""
    _payload(recv_o, "recv_o", 5)
    W, W2, T, Hc, D = recv_o.shape
    if W2 != W:
        raise ValueError("recv_o must be [W, W, T, Hc, D], got %s" % (tuple(recv_o.shape),))
    _expect(recv_lse, "recv_lse", (W, W, T, Hc), torch.float32, recv_o.device)
    if out is None:
        out = torch.empty((W, T, Hc, D), dtype=recv_o.dtype, device=recv_o.device)
    if out_lse is None:
        out_lse = torch.empty((W, T, Hc), dtype=torch.float32, device=recv_o.device)
    _expect(out, "out", (W, T, Hc, D), recv_o.dtype, recv_o.device)
    _expect(out_lse, "out_lse", (W, T, Hc), torch.float32, recv_o.device)
    for t, n in ((recv_o, "recv_o"), (recv_lse, "recv_lse"), (out, "out"), (out_lse, "out_lse")):
        _dense(t, n)
    _check(_lib.cp_lse_combine(_ptr(recv_o), _ptr(recv_lse), W, T, Hc, D, _dtype(recv_o),
                               _ptr(out), _ptr(out_lse), _stream(stream)))
    return out, out_lse


def cp_pack_permute_combine_fused(o: torch.Tensor, smax: torch.Tensor, ssum: torch.Tensor,
                                  out: Optional[torch.Tensor] = None,
                                  out_lse: Optional[torch.Tensor] = None, scatter_dim: int = 1,
                                  stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Head chunks (scatter_dim=1): out [W, T, H/W, D], out_lse [W, T, H/W].
    Token chunks (scatter_dim=0): out [W, T/W, H, D], out_lse [W, T/W, H]."""
    _payload(o, "o", 4)
    W, T, H, D = o.shape
    _stats(o, smax, ssum)
    shape = _packet_shape(W, T, H, scatter_dim)[1:]
    if out is None:
        out = torch.empty(shape + (D,), dtype=o.dtype, device=o.device)
    if out_lse is None:
        out_lse = torch.empty(shape, dtype=torch.float32, device=o.device)
    _expect(out, "out", shape + (D,), o.dtype, o.device)
    _expect(out_lse, "out_lse", shape, torch.float32, o.device)
    _dense(out, "out")
    _dense(out_lse, "out_lse")
    _check(_lib.cp_pack_permute_combine_fused(_ptr(o), _strides3(o), _ptr(smax), _strides3(smax),
                                              _ptr(ssum), _strides3(ssum), W, T, H, D, _dtype(o),
                                              scatter_dim, _ptr(out), _ptr(out_lse),
                                              _stream(stream)))
    return out, out_lse


# ---- one process per GPU: the exchange across W real ranks ------------------------------------

def _strides_plane(t) -> Strides3:
    """Strides of one rank's [T, H] or [T, H, D] plane (the rank stride is unused)."""
    st = t.stride()
    if t.dim() == 3 and st[2] != 1:
        raise ValueError("the head dim (last) of o must be contiguous")
    return Strides3(0, st[0], st[1])


def cp_pack_lse_rank(o: torch.Tensor, smax: torch.Tensor, ssum: torch.Tensor, W: int,
                     scatter_dim: int = 1, pkt_o: Optional[torch.Tensor] = None,
                     pkt_lse: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's send packet for W destinations: o [T, H, D], smax/ssum [T, H]
    -> pkt_o [W, T, H/W, D], pkt_lse [W, T, H/W] (heads) or [W, T/W, H, D],
    [W, T/W, H] (tokens); block j goes to destination j."""
    _payload(o, "o", 3)
    T, H, D = o.shape
    _expect(smax, "smax", (T, H), torch.float32, o.device)
    _expect(ssum, "ssum", (T, H), torch.float32, o.device)
    shape = _packet_shape(W, T, H, scatter_dim)[1:]        # [W_dst, rows...]
    if pkt_o is None:
        pkt_o = torch.empty(shape + (D,), dtype=o.dtype, device=o.device)
    if pkt_lse is None:
        pkt_lse = torch.empty(shape, dtype=torch.float32, device=o.device)
    _expect(pkt_o, "pkt_o", shape + (D,), o.dtype, o.device)
    _expect(pkt_lse, "pkt_lse", shape, torch.float32, o.device)
    _dense(pkt_o, "pkt_o")
    _dense(pkt_lse, "pkt_lse")
    _check(_lib.cp_pack_lse_rank(_ptr(o), _strides_plane(o), _ptr(smax), _strides_plane(smax),
                                 _ptr(ssum), _strides_plane(ssum), W, T, H, D, _dtype(o),
                                 scatter_dim, _ptr(pkt_o), _ptr(pkt_lse), _stream(stream)))
    return pkt_o, pkt_lse


def cp_lse_combine_rank(recv_o: torch.Tensor, recv_lse: torch.Tensor,
                        out: Optional[torch.Tensor] = None, out_lse: Optional[torch.Tensor] = None,
                        stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One destination's combine: recv_o [W, T, Hc, D], recv_lse [W, T, Hc]
    -> out [T, Hc, D], out_lse [T, Hc] (token chunks: T/W as T, H as Hc)."""
    _payload(recv_o, "recv_o", 4)
    W, T, Hc, D = recv_o.shape
    _expect(recv_lse, "recv_lse", (W, T, Hc), torch.float32, recv_o.device)
    if out is None:
        out = torch.empty((T, Hc, D), dtype=recv_o.dtype, device=recv_o.device)
    if out_lse is None:
        out_lse = torch.empty((T, Hc), dtype=torch.float32, device=recv_o.device)
    _expect(out, "out", (T, Hc, D), recv_o.dtype, recv_o.device)
    _expect(out_lse, "out_lse", (T, Hc), torch.float32, recv_o.device)
    for t, n in ((recv_o, "recv_o"), (recv_lse, "recv_lse"), (out, "out"), (out_lse, "out_lse")):
        _dense(t, n)
    _check(_lib.cp_lse_combine_rank(_ptr(recv_o), _ptr(recv_lse), W, T, Hc, D, _dtype(recv_o),
                                    _ptr(out), _ptr(out_lse), _stream(stream)))
    return out, out_lse


def cp_pull_combine(o: Sequence, smax: Sequence, ssum: Sequence, dst: int, scatter_dim: int = 1,
                    out: Optional[torch.Tensor] = None, out_lse: Optional[torch.Tensor] = None,
                    device: Optional[torch.device] = None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Destination `dst` of W real ranks, pulled straight from every rank's
    planes: o[r] [T, H, D], smax[r]/ssum[r] [T, H], all with the same strides.
    A plane is a tensor of this device or any object with ``shape``, ``dtype``,
    ``stride()`` and ``data_ptr()`` giving an address this device can read (a
    peer's buffer mapped into this process). Returns out [T, H/W, D],
    out_lse [T, H/W] (heads) or [T/W, H, D], [T/W, H] (tokens), on `device`
    (default: the current device)."""
    W = len(o)
    if W < 1 or len(smax) != W or len(ssum) != W:
        raise ValueError("o, smax and ssum must list the same W >= 1 ranks")
    T, H, D = _plane(o[0], "o[0]", 3, None)
    for r in range(W):
        _plane(o[r], "o[%d]" % r, 3, o[0])
        _plane(smax[r], "smax[%d]" % r, 2, smax[0], (T, H))
        _plane(ssum[r], "ssum[%d]" % r, 2, ssum[0], (T, H))
    if o[0].dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("payload dtype must be bfloat16 or float16, got %s" % o[0].dtype)
    if smax[0].dtype != torch.float32 or ssum[0].dtype != torch.float32:
        raise ValueError("smax and ssum must be float32")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    shape = _packet_shape(W, T, H, scatter_dim)[2:]
    if out is None:
        out = torch.empty(shape + (D,), dtype=o[0].dtype, device=dev)
    if out_lse is None:
        out_lse = torch.empty(shape, dtype=torch.float32, device=dev)
    _expect(out, "out", shape + (D,), o[0].dtype, dev)
    _expect(out_lse, "out_lse", shape, torch.float32, dev)
    _dense(out, "out")
    _dense(out_lse, "out_lse")
    po = (ctypes.c_void_p * W)(*[t.data_ptr() for t in o])
    pm = (ctypes.c_void_p * W)(*[t.data_ptr() for t in smax])
    ps = (ctypes.c_void_p * W)(*[t.data_ptr() for t in ssum])
    _check(_lib.cp_pull_combine(po, _strides_plane(o[0]), pm, _strides_plane(smax[0]), ps,
                                _strides_plane(ssum[0]), W, T, H, D, _dtype(o[0]), scatter_dim,
                                dst, _ptr(out), _ptr(out_lse), _stream(stream)))
    return out, out_lse


def _plane(t, name: str, ndim: int, like, shape=None):
    """Shape (and, against `like`, dtype and strides) of one rank's plane."""
    got = tuple(t.shape)
    if len(got) != ndim:
        raise ValueError("%s must have %d dimensions, got shape %s" % (name, ndim, got))
    if shape is not None and got != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, got, tuple(shape)))
    if like is not None:
        if got != tuple(like.shape) or t.dtype != like.dtype:
            raise ValueError("%s differs from the first rank's plane in shape or dtype" % name)
        if tuple(t.stride()) != tuple(like.stride()):
            raise ValueError("%s has other strides than the first rank's plane" % name)
    return got


def ulysses_seq2head(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """x [W, B, S/W, H, D] (contiguous) -> [W, B, S, H/W, D]."""
    if not isinstance(x, torch.Tensor) or x.dim() != 5:
        raise ValueError("x must be a [W, B, S/W, H, D] tensor")
    W, B, S_l, H, D = x.shape
    shape = (W, B, S_l * W, _split(H, W, "H"), D)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    _expect(out, "out", shape, x.dtype, x.device)
    _dense(x, "x")
    _dense(out, "out")
    _check(_lib.ulysses_seq2head(_ptr(x), _ptr(out), W, B, S_l, H, D, x.element_size(),
                                 _stream(stream)))
    return out


def ulysses_head2seq(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """x [W, B, S, Hc, D] (contiguous) -> [W, B, S/W, Hc*W, D]."""
    if not isinstance(x, torch.Tensor) or x.dim() != 5:
        raise ValueError("x must be a [W, B, S, H/W, D] tensor")
    W, B, S, Hc, D = x.shape
    shape = (W, B, _split(S, W, "S"), Hc * W, D)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    _expect(out, "out", shape, x.dtype, x.device)
    _dense(x, "x")
    _dense(out, "out")
    _check(_lib.ulysses_head2seq(_ptr(x), _ptr(out), W, B, S // W, Hc * W, D, x.element_size(),
                                 _stream(stream)))
    return out


def _ulysses_pull(x: Sequence, out_shape, out: Optional[torch.Tensor], device):
    """Checks of the W ranks' tensors (same shape, dtype, contiguous) and the
    output; returns the output and the table of the ranks' addresses."""
    W = len(x)
    for r in range(W):
        _plane(x[r], "x[%d]" % r, 4, x[0])
        if not _is_dense(x[r]):
            raise ValueError("x[%d] must be contiguous" % r)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    if out is None:
        out = torch.empty(out_shape, dtype=x[0].dtype, device=dev)
    _expect(out, "out", out_shape, x[0].dtype, dev)
    _dense(out, "out")
    return out, (ctypes.c_void_p * W)(*[t.data_ptr() for t in x])


def _is_dense(t) -> bool:
    shape, st, want = tuple(t.shape), tuple(t.stride()), 1
    for n, s in zip(reversed(shape), reversed(st)):
        if n != 1 and s != want:
            return False
        want *= n
    return True


def ulysses_seq2head_pull(x: Sequence, dst: int, out: Optional[torch.Tensor] = None,
                          device: Optional[torch.device] = None, stream=None) -> torch.Tensor:
    """Destination `dst` of the seq->head all-to-all across W real ranks: x[r]
    [B, S/W, H, D] (this device's tensor or a peer's mapped into this process)
    -> out [B, S, H/W, D]."""
    W = len(x)
    if W < 1:
        raise ValueError("x must list W >= 1 ranks")
    B, S_l, H, D = x[0].shape
    out, tab = _ulysses_pull(x, (B, S_l * W, _split(H, W, "H"), D), out, device)
    _check(_lib.ulysses_seq2head_pull(tab, _ptr(out), W, B, S_l, H, D, out.element_size(), dst,
                                      _stream(stream)))
    return out


def ulysses_head2seq_pull(x: Sequence, dst: int, out: Optional[torch.Tensor] = None,
                          device: Optional[torch.device] = None, stream=None) -> torch.Tensor:
    """Destination `dst` of the head->seq all-to-all across W real ranks: x[r]
    [B, S, H/W, D] -> out [B, S/W, H, D]."""
    W = len(x)
    if W < 1:
        raise ValueError("x must list W >= 1 ranks")
    B, S, Hc, D = x[0].shape
    S_l = _split(S, W, "S")
    out, tab = _ulysses_pull(x, (B, S_l, Hc * W, D), out, device)
    _check(_lib.ulysses_head2seq_pull(tab, _ptr(out), W, B, S_l, Hc * W, D, out.element_size(),
                                      dst, _stream(stream)))
    return out


class _SeqToHead(torch.autograd.Function):
    """all_to_all_4D(x, 2, 1) with its adjoint: the gradient of a layout
    permutation is the inverse permutation of the incoming gradient."""

    @staticmethod
    def forward(ctx, x):
        return ulysses_seq2head(x.contiguous())

    @staticmethod
    def backward(ctx, g):
        return ulysses_head2seq(g.contiguous())


class _HeadToSeq(torch.autograd.Function):
    """all_to_all_4D(x, 1, 2) with its adjoint (seq -> head of the gradient)."""

    @staticmethod
    def forward(ctx, x):
        return ulysses_head2seq(x.contiguous())

    @staticmethod
    def backward(ctx, g):
        return ulysses_seq2head(g.contiguous())


def ulysses_seq2head_autograd(x: torch.Tensor) -> torch.Tensor:
    """ulysses_seq2head that autograd differentiates (backward: ulysses_head2seq)."""
    return _SeqToHead.apply(x)


def ulysses_head2seq_autograd(x: torch.Tensor) -> torch.Tensor:
    """ulysses_head2seq that autograd differentiates (backward: ulysses_seq2head)."""
    return _HeadToSeq.apply(x)
