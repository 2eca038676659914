"""The C ABI without a GPU: the library builds and loads, exports every symbol
include/kla.h declares, and rejects invalid requests on the host before any
launch."""
import ctypes
import os
import re

import pytest

from bayesian_filter_scan_b200 import build as kbuild
from bayesian_filter_scan_b200 import kla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kla.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "kla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kla_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert "kla_forward" in names and "kla_precision" in names
    for n in names:
        assert hasattr(L, n), n
    assert sorted(kla.EXPORTS) == names


def test_version_and_status_strings(L):
    assert L.kla_version() >= 100
    for s in range(6):
        assert kla.status_string(s)


def _desc(**kw):
    d = dict(B=1, T=64, H=2, dk=64, dv=64, dtype=kla.KLA_BF16, mode=kla.KLA_DIAG)
    d.update(kw)
    return kla.make_desc(**d)


def _fwd(L, desc, ptrs=None, ws=None, ws_bytes=0):
    p = ptrs if ptrs is not None else [ctypes.c_void_p(4096 * (i + 1)) for i in range(7)]
    q, k, v, a, qn, beta, out = p
    return L.kla_forward(ctypes.byref(desc), q, k, v, a, qn, beta, None, None, out, None, None,
                         ws, ws_bytes, None)


@pytest.mark.parametrize("bad", [dict(dk=48), dict(dk=256), dict(dv=8), dict(H=0), dict(B=-1),
                                 dict(dtype=7), dict(mode=3), dict(dv=512)])
def test_invalid_descriptors_are_rejected(L, bad):
    desc = _desc(**bad)
    assert _fwd(L, desc) == kla.KLA_ERR_INVALID_ARG
    assert L.kla_workspace_bytes(ctypes.byref(desc)) == 0


def test_null_and_misaligned_pointers_are_rejected(L):
    desc = _desc()
    ptrs = [ctypes.c_void_p(4096 * (i + 1)) for i in range(7)]
    ptrs[2] = None
    assert _fwd(L, desc, ptrs) == kla.KLA_ERR_INVALID_ARG
    ptrs = [ctypes.c_void_p(4096 * (i + 1)) for i in range(7)]
    ptrs[3] = ctypes.c_void_p(4096 * 4 + 4)
    assert _fwd(L, desc, ptrs) == kla.KLA_ERR_INVALID_ARG
    assert L.kla_forward(None, *([None] * 11), None, 0, None) == kla.KLA_ERR_INVALID_ARG


def test_empty_input_is_a_noop(L):
    desc = _desc(T=0)
    assert _fwd(L, desc, [None] * 7) == kla.KLA_OK


def test_workspace_size_and_check(L):
    # long rows with few heads need the segmented path and its workspace
    desc = _desc(B=1, T=131072, H=16, dk=128, dv=128)
    n = L.kla_workspace_bytes(ctypes.byref(desc))
    assert n > 0 and n % 256 == 0
    # too small a workspace is refused before any launch
    assert _fwd(L, desc, ws=ctypes.c_void_p(1 << 20), ws_bytes=n - 256) == kla.KLA_ERR_INVALID_ARG
    # misaligned workspace too
    assert _fwd(L, desc, ws=ctypes.c_void_p((1 << 20) + 16), ws_bytes=n) == kla.KLA_ERR_INVALID_ARG
    # the precision API always scans, so it needs a workspace for unpacked rows
    assert L.kla_precision_workspace_bytes(ctypes.byref(_desc())) > 0


def test_decode_step_requires_single_token(L):
    desc = _desc(T=2)
    r = L.kla_decode_step(ctypes.byref(desc), *[ctypes.c_void_p(4096 * (i + 1)) for i in range(9)],
                          ctypes.c_void_p(4096 * 20), None)
    assert r == kla.KLA_ERR_INVALID_ARG


def test_host_buffer_size_covers_inputs_outputs_and_workspace(L):
    desc = _desc(B=2, T=1000, H=4, dk=64, dv=128)
    n = L.kla_host_device_bytes(ctypes.byref(desc))
    ntok = 2000
    io = ntok * 4 * (64 * 2 * 2 + 128 * 2 * 2 + 64 * 4 * 2 + 4)
    assert n >= io + L.kla_workspace_bytes(ctypes.byref(desc))


class _FakePtr:
    """A stand-in for a device tensor: the plan reads only the descriptor's
    shapes, never the packed-sequence offsets themselves."""

    def data_ptr(self):
        return 256


@pytest.mark.parametrize("shape,expect", [
    # (B, T, H, dk, dv, dtype, mode, packed sequences) -> (segments per row, launches, tensor cores)
    ((4, 2048, 8, 64, 64, kla.KLA_BF16, kla.KLA_DIAG, 0), (8, 4, True)),      # small layer: 256 CTAs, two per SM
    ((8, 4096, 16, 128, 128, kla.KLA_BF16, kla.KLA_DIAG, 0), (1, 1, True)),   # 1.3B layer: rows fill the SMs
    ((1, 131072, 16, 128, 128, kla.KLA_BF16, kla.KLA_DIAG, 0), (9, 5, True)),  # long context: separate carry
    ((2, 16384, 32, 64, 128, kla.KLA_BF16, kla.KLA_ISO, 8), (1, 2, True)),   # packed: length ranking + walk
    ((1, 9000, 2, 64, 64, kla.KLA_BF16, kla.KLA_DIAG, 1700), (1, 1, True)),  # > 1024 sequences: input order
    # 128 blocks, room for 74 CTAs per row x head: 64 segments of 2 blocks; 126
    # blocks before the last segment, so the Moebius carry is its own launch
    ((1, 8192, 2, 64, 128, kla.KLA_BF16, kla.KLA_DIAG, 0), (64, 5, True)),
    ((1, 256, 2, 16, 16, kla.KLA_FP32, kla.KLA_DIAG, 0), (4, 5, False)),      # fp32: CUDA-core walk passes
])
def test_launch_plan_of_the_workloads(L, shape, expect):
    # on a host without a GPU the plan assumes the 148 SMs of a B200
    B, T, H, dk, dv, dt, mode, nseq = shape
    d = kla.make_desc(B, T, H, dk, dv, dt, mode, _FakePtr() if nseq else None, nseq)
    p = kla.plan(d)
    assert (p["segments"], p["launches"], p["tensor_core"]) == expect


def test_backward_host_validation(L):
    desc = _desc(B=2, T=100, H=4, dk=64, dv=128)
    n = L.kla_backward_workspace_bytes(ctypes.byref(desc))
    # per token-head: lambda, gate, dL/dlambda (dk each), dq^, dk^, G (dk each), 3 head scalars;
    # per unit: the final-state gate term (dk)
    assert n >= 4 * (2 * 100 * 4 * (6 * 64 + 3) + 8 * 64) and n % 256 == 0
    p = [ctypes.c_void_p(4096 * (i + 1)) for i in range(19)]
    ws = ctypes.c_void_p(1 << 24)
    assert L.kla_backward(ctypes.byref(desc), *p, ws, n - 256, None) == kla.KLA_ERR_INVALID_ARG
    q = list(p)
    q[0] = None                     # q
    assert L.kla_backward(ctypes.byref(desc), *q, ws, n, None) == kla.KLA_ERR_INVALID_ARG
    q = list(p)
    q[8] = ctypes.c_void_p(4096 * 9 + 4)   # dout must be 16-byte aligned
    assert L.kla_backward(ctypes.byref(desc), *q, ws, n, None) == kla.KLA_ERR_INVALID_ARG
    # dv = 256 is forward-only
    wide = _desc(dv=256)
    assert L.kla_backward_workspace_bytes(ctypes.byref(wide)) == 0
    assert L.kla_backward(ctypes.byref(wide), *p, ws, n, None) == kla.KLA_ERR_UNSUPPORTED
    # an empty input launches nothing
    assert L.kla_backward(ctypes.byref(_desc(T=0)), *([None] * 19), None, 0, None) == kla.KLA_OK
