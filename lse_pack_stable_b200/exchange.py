"""The DCP exchange across real ranks: one process per GPU, torch.distributed
for the plumbing, this package's kernels for every step of the data path.

Partitioning (vLLM-Ascend pull request "Fuse local SFA LSE formation into DCP
pack", section "What this PR does / why we need it?": pack -> all-to-all ->
stable combine): rank r holds the partial attention output of KV shard r,
o [T, H, D] with its fp32 softmax max and sum [T, H]. Destination j receives
head chunk j (heads j*Hc .. (j+1)*Hc - 1, Hc = H / W) of every rank -- or,
with scatter_dim = 0, token chunk j (tokens j*T/W ..) with all heads -- and
merges the W contributions with the stable log-sum-exp combine.

Two ways across, both giving rank j destination j's block of the single-GPU
fused result, bit for bit:

* ``A2aExchange``: ``cp_pack_lse_rank`` writes this rank's send packet (payload
  region, LSE region; block j for destination j), one all-to-all per region
  moves the blocks (NCCL over NVLink), ``cp_lse_combine_rank`` merges what
  arrived.
* ``PullExchange``: every rank's o/max/sum planes live in buffers mapped into
  every other rank's process (``cp_ipc_export`` / ``cp_ipc_import``: plain
  CUDA IPC, no multicast); ``cp_pull_combine`` on rank j reads the rows it
  merges straight from each owner's HBM, so no packet exists. A one-element
  all-reduce before the kernel (every owner has written its planes) and after
  it (no owner overwrites them while a peer still reads) orders it against
  the other ranks on the stream, with no host synchronisation and no
  device-side wait in any kernel of this package.

``UlyssesPullExchange`` does the same for the Ulysses layout all-to-alls: each
rank's sequence shard and head shard are mapped into every rank, and
destination j's seq->head (head->seq) result is read out of all of them by
``ulysses_seq2head_pull`` (``ulysses_head2seq_pull``).
"""
from __future__ import annotations

import ctypes
from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist

from . import (CplseError, IpcHandle, _check, _lib, cp_lse_combine_rank, cp_pack_lse_rank,
               cp_pull_combine, ulysses_head2seq_pull, ulysses_seq2head_pull)


def ipc_export(t: torch.Tensor) -> bytes:
    """The bytes another process of this node needs to map `t` (a CUDA tensor
    of the current device, allocated by torch's caching allocator)."""
    h = IpcHandle()
    _check(_lib.cp_ipc_export(t.data_ptr(), ctypes.byref(h)))
    return bytes(h)


def ipc_import(blob: bytes) -> Tuple[int, int]:
    """Map another process's buffer: returns (base, address); the address is
    usable by this process's kernels on the current device until
    ``ipc_close(base)``."""
    h = IpcHandle.from_buffer_copy(blob)
    base, p = ctypes.c_void_p(), ctypes.c_void_p()
    _check(_lib.cp_ipc_import(ctypes.byref(h), ctypes.byref(base), ctypes.byref(p)))
    return base.value, p.value


def ipc_close(base: int) -> None:
    _check(_lib.cp_ipc_close(base))


class _Plane:
    """A peer rank's plane as the binding sees one: shape, dtype, strides and
    an address in this process (duck-typed for cp_pull_combine)."""

    def __init__(self, addr: int, like: torch.Tensor):
        self._addr, self.shape, self.dtype = addr, like.shape, like.dtype
        self._stride = like.stride()
        self.device = like.device

    def data_ptr(self) -> int:
        return self._addr

    def stride(self):
        return self._stride

    def dim(self) -> int:
        return len(self.shape)


def _plane_shape(W: int, T: int, H: int, scatter_dim: int):
    if H % W:
        raise ValueError("H = %d is not a multiple of W = %d" % (H, W))
    if scatter_dim == 1:
        return (T, H // W)
    if scatter_dim == 0:
        if T % W:
            raise ValueError("T = %d is not a multiple of W = %d" % (T, W))
        return (T // W, H)
    raise ValueError("scatter_dim must be 0 or 1")


class A2aExchange:
    """pack -> all-to-all (one per packet region) -> combine, for this rank.

    The send and receive packets are allocated once here and reused by every
    call. ``pack`` and ``combine`` default to the CUDA kernels; they are
    parameters only so that the collective plumbing can be exercised with
    other implementations of the same contracts."""

    def __init__(self, T: int, H: int, D: int, dtype: torch.dtype, device,
                 group: Optional[dist.ProcessGroup] = None, scatter_dim: int = 1,
                 pack: Callable = cp_pack_lse_rank, combine: Callable = cp_lse_combine_rank):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.T, self.H, self.D, self.scatter_dim = T, H, D, scatter_dim
        rows = _plane_shape(self.W, T, H, scatter_dim)
        shape = (self.W,) + rows
        self.send_o = torch.empty(shape + (D,), dtype=dtype, device=device)
        self.send_lse = torch.empty(shape, dtype=torch.float32, device=device)
        self.recv_o = torch.empty_like(self.send_o)
        self.recv_lse = torch.empty_like(self.send_lse)
        self._pack, self._combine = pack, combine

    def __call__(self, o: torch.Tensor, smax: torch.Tensor, ssum: torch.Tensor,
                 out: Optional[torch.Tensor] = None, out_lse: Optional[torch.Tensor] = None):
        """o [T, H, D], smax/ssum [T, H] of this rank -> this destination's
        out [T, H/W, D] and out_lse [T, H/W] (token chunks: [T/W, H, D], [T/W, H])."""
        self._pack(o, smax, ssum, self.W, scatter_dim=self.scatter_dim, pkt_o=self.send_o,
                   pkt_lse=self.send_lse)
        # block j of each region goes to rank j; a bit copy, so the payload moves as bytes
        dist.all_to_all_single(self.recv_o.view(torch.uint8), self.send_o.view(torch.uint8),
                               group=self.group)
        dist.all_to_all_single(self.recv_lse, self.send_lse, group=self.group)
        return self._combine(self.recv_o, self.recv_lse, out=out, out_lse=out_lse)


def _stream_barrier(flag: torch.Tensor, group, stream=None) -> None:
    """Every rank of `group` reaches this point on `stream` before anything
    enqueued on `stream` afterwards runs: a one-element all-reduce issued with
    `stream` current (torch orders a collective after the current stream's
    work and makes that stream wait for it)."""
    if stream is None:
        dist.all_reduce(flag, group=group)
        return
    with torch.cuda.stream(stream):
        dist.all_reduce(flag, group=group)


class PeerMapError(RuntimeError):
    """Some rank of the group could not share or map the buffers; every rank
    raises it at the same point, so that none is left waiting in a collective."""


class PeerMap:
    """Tensors of this rank shared with every rank of the group: ``table(i)[r]``
    is rank r's tensor i -- this rank's own tensor, or the peer's mapped into
    this process (a ``_Plane``). Construction and ``close`` are collective.

    The outcome is the group's, not this rank's: a failed export shows in the
    gathered handles, a failed import in one all-reduce of a success flag, and
    then every rank unmaps what it had mapped and raises ``PeerMapError``."""

    def __init__(self, tensors, group: Optional[dist.ProcessGroup] = None):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = tensors[0].device
        err: Optional[Exception] = None
        try:
            mine = [ipc_export(t) for t in tensors]
        except CplseError as e:
            mine, err = None, e
        every: List = [None] * self.W
        dist.all_gather_object(every, mine, group=group)
        self._bases: List[int] = []
        self._tables: List[List] = [[] for _ in tensors]
        failed = [r for r in range(self.W) if every[r] is None]
        if failed:
            raise PeerMapError("rank(s) %s could not export their buffers%s"
                               % (failed, ": %s" % err if err is not None else ""))
        for r in range(self.W):
            for i, t in enumerate(tensors):
                if r == self.rank:
                    self._tables[i].append(t)
                elif err is None:
                    try:
                        base, addr = ipc_import(every[r][i])
                    except CplseError as e:
                        err = e
                        continue
                    self._bases.append(base)
                    self._tables[i].append(_Plane(addr, t))
        ok = torch.tensor([0.0 if err is not None else 1.0], device=self.device)
        dist.all_reduce(ok, op=dist.ReduceOp.MIN, group=group)
        if ok.item() < 1.0:
            self._unmap()
            raise PeerMapError("mapping a peer's buffers failed on %s"
                               % ("this rank: %s" % err if err is not None else "another rank"))

    def table(self, i: int) -> List:
        return self._tables[i]

    def _unmap(self) -> None:
        err = None
        for b in self._bases:
            try:
                ipc_close(b)
            except CplseError as e:  # keep closing the others
                err = e
        self._bases = []
        if err is not None:
            raise err

    def close(self) -> None:
        """Unmap the peers' tensors, once every rank has finished reading."""
        if not self._bases:
            return
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        self._unmap()


class PullExchange:
    """This rank's o/max/sum planes, mapped into every rank's process, and the
    pull kernel that merges destination `rank`'s rows from all of them.

    The producer writes this rank's partial output into ``o``, ``smax`` and
    ``ssum`` (allocated here); each call then returns this destination's
    combined rows. Construction is collective (every rank of the group), and
    so is ``close()``, which every rank calls before dropping the object: the
    planes stay allocated until then, as peers may still read them."""

    def __init__(self, T: int, H: int, D: int, dtype: torch.dtype, device,
                 group: Optional[dist.ProcessGroup] = None, scatter_dim: int = 1):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = torch.device(device)
        self.scatter_dim = scatter_dim
        self.out_rows = _plane_shape(self.W, T, H, scatter_dim)
        self.o = torch.empty((T, H, D), dtype=dtype, device=device)
        self.smax = torch.empty((T, H), dtype=torch.float32, device=device)
        self.ssum = torch.empty((T, H), dtype=torch.float32, device=device)
        self._flag = torch.zeros(1, dtype=torch.float32, device=device)
        self.peers = PeerMap([self.o, self.smax, self.ssum], group)
        self.o_tab, self.m_tab, self.s_tab = (self.peers.table(i) for i in range(3))

    def barrier(self, stream=None) -> None:
        """Barrier of the group, ordered on `stream` (default: the current
        stream): a one-element all-reduce issued from that stream."""
        _stream_barrier(self._flag, self.group, stream)

    def __call__(self, out: Optional[torch.Tensor] = None,
                 out_lse: Optional[torch.Tensor] = None, stream=None):
        self.barrier(stream)    # every rank has written its planes
        res = cp_pull_combine(self.o_tab, self.m_tab, self.s_tab, self.rank,
                              scatter_dim=self.scatter_dim, out=out, out_lse=out_lse,
                              device=self.device, stream=stream)
        self.barrier(stream)    # no rank overwrites its planes while a peer reads them
        return res

    def close(self) -> None:
        self.peers.close()


class UlyssesPullExchange:
    """The Ulysses all-to-alls across real ranks as load/store over NVLink
    (FastVideo "[perf] Probe H3 chunked all-to-all with direct output slices":
    all_to_all_4D(x, 2, 1) and its inverse, byte-identical to the NCCL path).

    This rank's sequence shard ``seq`` [B_seq, S/W, H, D] (what seq->head
    scatters by heads) and head shard ``head`` [B_head, S, H/W, D] (what
    head->seq gathers back) are allocated here and mapped into every rank;
    ``seq2head()`` returns this rank's [B_seq, S, H/W, D], ``head2seq()`` its
    [B_head, S/W, H, D]. Construction is collective."""

    def __init__(self, B_seq: int, B_head: int, S: int, H: int, D: int, dtype: torch.dtype,
                 device, group: Optional[dist.ProcessGroup] = None):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = torch.device(device)
        S_l = S // self.W
        if S_l * self.W != S or H % self.W:
            raise ValueError("S = %d and H = %d must be multiples of W = %d" % (S, H, self.W))
        self.seq = torch.empty((B_seq, S_l, H, D), dtype=dtype, device=device)
        self.head = torch.empty((B_head, S, H // self.W, D), dtype=dtype, device=device)
        self._flag = torch.zeros(1, dtype=torch.float32, device=device)
        self.peers = PeerMap([self.seq, self.head], group)

    def barrier(self, stream=None) -> None:
        _stream_barrier(self._flag, self.group, stream)

    def seq2head(self, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        self.barrier(stream)
        res = ulysses_seq2head_pull(self.peers.table(0), self.rank, out=out, device=self.device,
                                    stream=stream)
        self.barrier(stream)
        return res

    def head2seq(self, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        self.barrier(stream)
        res = ulysses_head2seq_pull(self.peers.table(1), self.rank, out=out, device=self.device,
                                    stream=stream)
        self.barrier(stream)
        return res

    def close(self) -> None:
        self.peers.close()
