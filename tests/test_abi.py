"""The C-ABI library on the host: it loads, exports every entry point the header
declares, and rejects bad arguments with the documented status before any
launch (no GPU needed: these checks run before the library touches CUDA)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import lse_pack_stable_b200 as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cplse.h")
S = cp.Strides3
L = cp._lib


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"CPLSE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    assert set(declared_symbols()) == set(cp.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(cp.LIBRARY_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_only_declared_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", cp.LIBRARY_PATH], capture_output=True,
                         text=True, check=True).stdout
    text_syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert text_syms == set(declared_symbols())


def test_abi_version():
    assert cp.abi_version() == cp.ABI_VERSION == 4


# aligned fake addresses: host checks run before any pointer is dereferenced or queried
A = 1 << 20


def _pack(W=2, T=4, H=8, D=64, dt=0, sd=1, o=A, m=2 * A, s=3 * A, po=4 * A, pl=5 * A,
          so=None, sm=None, ss=None):
    so = so or S(T * H * D, H * D, D)
    sm = sm or S(T * H, H, 1)
    ss = ss or S(T * H, H, 1)
    return L.cp_pack_lse(o, so, m, sm, s, ss, W, T, H, D, dt, sd, po, pl, None)


def _fused(W=2, T=4, H=8, D=64, dt=0, o=A, m=2 * A, s=3 * A, out=4 * A, ol=5 * A, so=None, sd=1):
    so = so or S(T * H * D, H * D, D)
    return L.cp_pack_permute_combine_fused(o, so, m, S(T * H, H, 1), s, S(T * H, H, 1), W, T, H,
                                           D, dt, sd, out, ol, None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(W=0), cp.CP_ERR_ARG, "W must be"),
    (dict(W=33, H=66), cp.CP_ERR_UNSUPPORTED, "exceeds"),
    (dict(W=3), cp.CP_ERR_SHAPE, "multiple of W"),
    (dict(D=60), cp.CP_ERR_SHAPE, "multiple of 8"),
    (dict(D=1032), cp.CP_ERR_UNSUPPORTED, "exceeds"),
    (dict(dt=7), cp.CP_ERR_ARG, "dtype"),
    (dict(sd=2), cp.CP_ERR_ARG, "scatter_dim"),
    (dict(sd=0, T=5), cp.CP_ERR_SHAPE, "T % W"),
    (dict(T=-1), cp.CP_ERR_ARG, "T must be"),
    (dict(o=0), cp.CP_ERR_ARG, "o is NULL"),
    (dict(pl=0), cp.CP_ERR_ARG, "pkt_lse is NULL"),
    (dict(o=A + 8), cp.CP_ERR_ALIGN, "o is not 16-byte aligned"),
    (dict(po=4 * A + 4), cp.CP_ERR_ALIGN, "pkt_o is not 16-byte aligned"),
    (dict(m=2 * A + 2), cp.CP_ERR_ALIGN, "smax is not 4-byte aligned"),
    (dict(so=S(4 * 8 * 64, 8 * 64, 60)), cp.CP_ERR_ALIGN, "multiples of 8"),
    (dict(sm=S(-1, 8, 1)), cp.CP_ERR_ARG, ">= 0"),
    (dict(po=A + 64), cp.CP_ERR_ALIAS, "pkt_o overlaps input o"),
    (dict(pl=3 * A), cp.CP_ERR_ALIAS, "pkt_lse overlaps input ssum"),
    (dict(pl=4 * A + 16), cp.CP_ERR_ALIAS, "outputs pkt_o and pkt_lse overlap"),
])
def test_pack_rejects(kw, status, msg):
    assert _pack(**kw) == status
    assert msg in cp.last_error()


def _device_check_failed(name):
    msg = cp.last_error()
    return msg.startswith(name + " is not device memory") or msg.startswith(
        name + ": cudaPointerGetAttributes failed")


def test_valid_arguments_reach_the_device_check():
    # every host check passes; the first check that needs the driver rejects the
    # fake (host) address, on a CPU-only machine and on a GPU machine alike
    assert _pack() == cp.CP_ERR_ARG and _device_check_failed("o")
    assert _fused() == cp.CP_ERR_ARG and _device_check_failed("o")
    assert L.cp_a2a_local_permute(A, 2 * A, 2, 16, None) == cp.CP_ERR_ARG
    assert _device_check_failed("send")


def test_empty_problem_is_ok_without_pointers():
    assert _pack(T=0, o=0, m=0, s=0, po=0, pl=0) == cp.CP_OK
    assert _fused(T=0, o=0, m=0, s=0, out=0, ol=0) == cp.CP_OK
    assert L.cp_a2a_local_permute(None, None, 4, 0, None) == cp.CP_OK
    assert L.ulysses_seq2head(None, None, 2, 0, 4, 4, 8, 2, None) == cp.CP_OK


@pytest.mark.parametrize("kw,status,msg", [
    (dict(out=0), cp.CP_ERR_ARG, "out is NULL"),
    (dict(out=4 * A + 2), cp.CP_ERR_ALIGN, "out is not 16-byte aligned"),
    (dict(out=A), cp.CP_ERR_ALIAS, "out overlaps input o"),
    (dict(ol=A + 4), cp.CP_ERR_ALIAS, "out_lse overlaps input o"),
    (dict(W=64, H=64), cp.CP_ERR_UNSUPPORTED, "exceeds"),
    (dict(sd=2), cp.CP_ERR_ARG, "scatter_dim must be"),
    (dict(sd=0, T=5), cp.CP_ERR_SHAPE, "token scatter needs T % W == 0"),
    (dict(sd=0, out=A + 64), cp.CP_ERR_ALIAS, "out overlaps input o"),
    # o's span follows its strides: a large token stride reaches the output
    (dict(so=S(8, 3 * A // 2 // 3, 64)), cp.CP_ERR_ALIAS, "overlaps input o"),
])
def test_fused_rejects(kw, status, msg):
    assert _fused(**kw) == status
    assert msg in cp.last_error()


@pytest.mark.parametrize("args,status,msg", [
    ((A, 2 * A, 0, 16), cp.CP_ERR_ARG, "W must be"),
    ((A, 2 * A, 40, 16), cp.CP_ERR_UNSUPPORTED, "exceeds"),
    ((A, 2 * A, 2, -16), cp.CP_ERR_ARG, "block_bytes"),
    ((A, A + 32, 2, 16), cp.CP_ERR_ALIAS, "recv overlaps input send"),
    ((0, 2 * A, 2, 16), cp.CP_ERR_ARG, "send is NULL"),
])
def test_permute_rejects(args, status, msg):
    assert L.cp_a2a_local_permute(*args, None) == status
    assert msg in cp.last_error()


@pytest.mark.parametrize("args,status,msg", [
    ((A, 8 * A, 2, 3, 4, 5, 8, 2), cp.CP_ERR_SHAPE, "multiple of W"),
    ((A, 8 * A, 2, 3, 4, 4, 8, 3), cp.CP_ERR_ARG, "elem_bytes"),
    ((A, 8 * A, 2, -1, 4, 4, 8, 2), cp.CP_ERR_ARG, ">= 0"),
    ((A, A + 2, 2, 3, 4, 4, 8, 2), cp.CP_ERR_ALIAS, "out overlaps input in"),
    ((A, 8 * A, 2, 3, 4, 4, 0, 2), cp.CP_ERR_SHAPE, "D must be"),
])
def test_ulysses_rejects(args, status, msg):
    for f in (L.ulysses_seq2head, L.ulysses_head2seq):
        assert f(*args, None) == status
        assert msg in cp.last_error()


@pytest.mark.parametrize("args,status,msg", [
    ((A, 2 * A, 2, 4, 0, 64, 0, 4 * A, 5 * A), cp.CP_ERR_SHAPE, "Hc must be"),
    ((A, 2 * A, 2, 4, 4, 12, 0, 4 * A, 5 * A), cp.CP_ERR_SHAPE, "multiple of 8"),
    ((A, 2 * A, 2, 4, 4, 64, 0, A + 16, 5 * A), cp.CP_ERR_ALIAS, "out overlaps input recv_o"),
    ((A + 4, 2 * A, 2, 4, 4, 64, 0, 4 * A, 5 * A), cp.CP_ERR_ALIGN, "recv_o"),
])
def test_combine_rejects(args, status, msg):
    assert L.cp_lse_combine(*args, None) == status
    assert msg in cp.last_error()


def test_binding_rejects_noncontiguous_and_dtype():
    import torch
    o = torch.zeros((2, 4, 8, 64), dtype=torch.float32)
    with pytest.raises(TypeError):
        cp.cp_pack_permute_combine_fused(o, torch.zeros(2, 4, 8), torch.zeros(2, 4, 8),
                                         out=torch.zeros(2, 4, 4, 64), out_lse=torch.zeros(2, 4, 4))
    ob = torch.zeros((2, 4, 8, 128), dtype=torch.bfloat16)[..., ::2]
    with pytest.raises(ValueError):
        cp.cp_pack_permute_combine_fused(ob, torch.zeros(2, 4, 8), torch.zeros(2, 4, 8),
                                         out=torch.zeros(2, 4, 4, 64, dtype=torch.bfloat16),
                                         out_lse=torch.zeros(2, 4, 4))


# ---- the per-rank entry points of the exchange across real ranks


def _pack_rank(W=2, T=4, H=8, D=64, dt=0, sd=1, o=A, m=2 * A, s=3 * A, po=4 * A, pl=5 * A):
    return L.cp_pack_lse_rank(o, S(0, H * D, D), m, S(0, H, 1), s, S(0, H, 1), W, T, H, D, dt,
                              sd, po, pl, None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(W=3), cp.CP_ERR_SHAPE, "multiple of W"),
    (dict(sd=0, T=5), cp.CP_ERR_SHAPE, "T % W"),
    (dict(o=0), cp.CP_ERR_ARG, "o is NULL"),
    (dict(po=4 * A + 8), cp.CP_ERR_ALIGN, "pkt_o is not 16-byte aligned"),
    # one plane: T*H*D*2 = 4 KiB of o; the packet starting inside it overlaps
    (dict(po=A + 4096 - 16), cp.CP_ERR_ALIAS, "pkt_o overlaps input o"),
])
def test_pack_rank_rejects(kw, status, msg):
    assert _pack_rank(**kw) == status
    assert msg in cp.last_error()


def test_pack_rank_one_plane_spans():
    # a packet right after one plane (T*H*D*2 bytes) does not overlap it: only
    # one source plane is read, whatever W is
    assert _pack_rank(po=A + 4096) == cp.CP_ERR_ARG and _device_check_failed("o")
    assert _pack_rank(T=0, o=0, m=0, s=0, po=0, pl=0) == cp.CP_OK


@pytest.mark.parametrize("args,status,msg", [
    ((A, 2 * A, 2, 4, 0, 64, 0, 4 * A, 5 * A), cp.CP_ERR_SHAPE, "Hc must be"),
    ((A, 2 * A, 2, 4, 4, 64, 0, A + 16, 5 * A), cp.CP_ERR_ALIAS, "out overlaps input recv_o"),
    ((A, 2 * A, 2, 4, 4, 64, 0, 4 * A + 2, 5 * A), cp.CP_ERR_ALIGN, "out is not 16"),
])
def test_combine_rank_rejects(args, status, msg):
    assert L.cp_lse_combine_rank(*args, None) == status
    assert msg in cp.last_error()


def _table(*addrs):
    return (ctypes.c_void_p * len(addrs))(*addrs)


def _pull(W=2, T=4, H=8, D=64, dt=0, sd=1, dst=0, o=None, m=None, s=None, out=8 * A,
          ol=9 * A):
    o = o if o is not None else _table(*[A + r * (A // 4) for r in range(W)])
    m = m if m is not None else _table(*[2 * A + r * (A // 4) for r in range(W)])
    s = s if s is not None else _table(*[3 * A + r * (A // 4) for r in range(W)])
    return L.cp_pull_combine(o, S(0, H * D, D), m, S(0, H, 1), s, S(0, H, 1), W, T, H, D, dt, sd,
                             dst, out, ol, None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(dst=2), cp.CP_ERR_ARG, "dst = 2"),
    (dict(dst=-1), cp.CP_ERR_ARG, "dst = -1"),
    (dict(W=3), cp.CP_ERR_SHAPE, "multiple of W"),
    (dict(sd=0, T=5), cp.CP_ERR_SHAPE, "T % W"),
    (dict(o=_table(A, 0)), cp.CP_ERR_ARG, "o[1] is NULL"),
    (dict(s=_table(3 * A, 3 * A + 2)), cp.CP_ERR_ALIGN, "ssum[1] is not 4-byte aligned"),
    (dict(o=_table(A + 8, A + A // 4)), cp.CP_ERR_ALIGN, "o[0] is not 16-byte aligned"),
    (dict(out=A + A // 4 + 64), cp.CP_ERR_ALIAS, "out overlaps input o[r]"),
    (dict(ol=0), cp.CP_ERR_ARG, "out_lse is NULL"),
])
def test_pull_rejects(kw, status, msg):
    assert _pull(**kw) == status
    assert msg in cp.last_error()


def test_pull_null_tables_and_device_check():
    assert L.cp_pull_combine(None, S(0, 512, 64), None, S(0, 8, 1), None, S(0, 8, 1), 2, 4, 8,
                             64, 0, 1, 0, 8 * A, 9 * A, None) == cp.CP_ERR_ARG
    assert "o is NULL" in cp.last_error()
    # every host check passes; the driver check then refuses the fake addresses
    assert _pull() == cp.CP_ERR_ARG and _device_check_failed("out")


def test_ipc_calls_reject_bad_arguments():
    h = cp.IpcHandle()
    assert L.cp_ipc_export(None, ctypes.byref(h)) == cp.CP_ERR_ARG and "p is NULL" in cp.last_error()
    assert L.cp_ipc_export(A, None) == cp.CP_ERR_ARG and "h is NULL" in cp.last_error()
    # a host address: the driver query refuses it (no GPU here, or not device memory)
    assert L.cp_ipc_export(A, ctypes.byref(h)) == cp.CP_ERR_ARG
    base, p = ctypes.c_void_p(), ctypes.c_void_p()
    h.offset, h.alloc_bytes = 64, 64
    assert L.cp_ipc_import(ctypes.byref(h), ctypes.byref(base), ctypes.byref(p)) == cp.CP_ERR_ARG
    assert "outside" in cp.last_error()
    assert L.cp_ipc_import(None, ctypes.byref(base), ctypes.byref(p)) == cp.CP_ERR_ARG
    assert L.cp_ipc_close(None) == cp.CP_ERR_ARG


@pytest.mark.parametrize("kw,status,msg", [
    (dict(dst=2), cp.CP_ERR_ARG, "dst = 2"),
    (dict(H=5), cp.CP_ERR_SHAPE, "multiple of W"),
    (dict(B=70000), cp.CP_ERR_UNSUPPORTED, "65535"),
    (dict(eb=3), cp.CP_ERR_ARG, "elem_bytes"),
    (dict(ins=(A, 0)), cp.CP_ERR_ARG, "in[1] is NULL"),
    (dict(out=A + A // 4 + 16), cp.CP_ERR_ALIAS, "out overlaps input in[r]"),
])
def test_ulysses_pull_rejects(kw, status, msg):
    W, B, S_l, H, D, eb, dst = 2, kw.get("B", 1), 4, kw.get("H", 4), 8, kw.get("eb", 2), kw.get("dst", 0)
    ins = kw.get("ins", (A, A + A // 4))
    for f in (L.ulysses_seq2head_pull, L.ulysses_head2seq_pull):
        assert f(_table(*ins), kw.get("out", 4 * A), W, B, S_l, H, D, eb, dst, None) == status
        assert msg in cp.last_error()


def test_ulysses_pull_reaches_the_device_check():
    for f in (L.ulysses_seq2head_pull, L.ulysses_head2seq_pull):
        assert f(_table(A, A + A // 4), 4 * A, 2, 1, 4, 4, 8, 2, 1, None) == cp.CP_ERR_ARG
        assert _device_check_failed("out")
        assert f(None, None, 2, 0, 4, 4, 8, 2, 0, None) == cp.CP_OK   # no rows
