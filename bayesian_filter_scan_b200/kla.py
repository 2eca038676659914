"""Python binding of libkla (include/kla.h): argument marshalling only.

Every step of the forward pass runs in libkla's CUDA kernels; this module
allocates outputs and workspace with torch (device memory and streams are the
only things torch provides), checks dtypes and shapes, and calls the C ABI
through ctypes on the current CUDA stream. There is no fallback: if libkla.so
is missing or a call fails, it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkla.so")

KLA_OK, KLA_ERR_INVALID_ARG, KLA_ERR_UNSUPPORTED, KLA_ERR_CUDA, KLA_ERR_TIMEOUT, KLA_ERR_RANGE = range(6)
KLA_BF16, KLA_FP32 = 0, 1
KLA_DIAG, KLA_ISO = 0, 1
# KLA_NOALLOC_SCRATCH_BYTES of include/kla.h: the fixed scratch area of kla_forward_noalloc
NOALLOC_SCRATCH_BYTES = 32 << 20

# Every symbol include/kla.h declares.
EXPORTS = ("kla_workspace_bytes", "kla_precision_workspace_bytes", "kla_forward", "kla_forward_profiled",
           "kla_plan", "kla_precision",
           "kla_decode_step", "kla_host_device_bytes", "kla_forward_host", "kla_check",
           "kla_status_string", "kla_version", "kla_forward_noalloc", "kla_kdn_forward",
           "kla_prologue", "kla_backward_workspace_bytes", "kla_backward")


class KlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


class KlaDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("dtype", ctypes.c_int),
                ("mode", ctypes.c_int), ("cu_seqlens", ctypes.c_void_p), ("num_seqs", ctypes.c_int)]


_lib = None
_P = ctypes.c_void_p


def lib():
    """Load libkla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libkla.so not found at %s; run `python -m bayesian_filter_scan_b200.build`"
                               % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        D = ctypes.POINTER(KlaDesc)
        L.kla_workspace_bytes.argtypes = [D]
        L.kla_workspace_bytes.restype = ctypes.c_size_t
        L.kla_precision_workspace_bytes.argtypes = [D]
        L.kla_precision_workspace_bytes.restype = ctypes.c_size_t
        L.kla_forward.argtypes = [D] + [_P] * 11 + [_P, ctypes.c_size_t, _P]
        L.kla_forward.restype = ctypes.c_int
        L.kla_forward_profiled.argtypes = [D] + [_P] * 11 + [_P, ctypes.c_size_t, _P, _P]
        L.kla_forward_profiled.restype = ctypes.c_int
        L.kla_plan.argtypes = [D, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                               ctypes.POINTER(ctypes.c_int)]
        L.kla_plan.restype = ctypes.c_int
        L.kla_precision.argtypes = [D] + [_P] * 6 + [_P, ctypes.c_size_t, _P]
        L.kla_precision.restype = ctypes.c_int
        L.kla_decode_step.argtypes = [D] + [_P] * 9 + [_P]
        L.kla_decode_step.restype = ctypes.c_int
        L.kla_host_device_bytes.argtypes = [D]
        L.kla_host_device_bytes.restype = ctypes.c_size_t
        L.kla_forward_host.argtypes = [D] + [_P] * 11 + [_P, ctypes.c_size_t, _P]
        L.kla_forward_host.restype = ctypes.c_int
        L.kla_forward_noalloc.argtypes = [D] + [_P] * 11 + [_P]
        L.kla_forward_noalloc.restype = ctypes.c_int
        L.kla_kdn_forward.argtypes = [D] + [_P] * 11 + [_P]
        L.kla_kdn_forward.restype = ctypes.c_int
        L.kla_prologue.argtypes = [D, ctypes.c_int] + [_P] * 18 + [_P]
        L.kla_prologue.restype = ctypes.c_int
        L.kla_backward_workspace_bytes.argtypes = [D]
        L.kla_backward_workspace_bytes.restype = ctypes.c_size_t
        L.kla_backward.argtypes = [D] + [_P] * 19 + [_P, ctypes.c_size_t, _P]
        L.kla_backward.restype = ctypes.c_int
        L.kla_check.argtypes = [_P]
        L.kla_check.restype = ctypes.c_int
        L.kla_status_string.argtypes = [ctypes.c_int]
        L.kla_status_string.restype = ctypes.c_char_p
        L.kla_version.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().kla_status_string(int(s)).decode()


def _check(s: int, what: str):
    if s != KLA_OK:
        raise KlaError(s, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_desc(B, T, H, dk, dv, dtype=KLA_BF16, mode=KLA_DIAG, cu_seqlens=None, num_seqs=0) -> KlaDesc:
    return KlaDesc(int(B), int(T), int(H), int(dk), int(dv), int(dtype), int(mode),
                   None if cu_seqlens is None else ctypes.c_void_p(cu_seqlens.data_ptr()), int(num_seqs))


def _desc_from(q, v, B, T, mode, cu_seqlens):
    Ntok, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype == torch.bfloat16:
        dt = KLA_BF16
    elif q.dtype == torch.float32:
        dt = KLA_FP32
    else:
        raise TypeError("q, k, v must be bfloat16 or float32")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
            raise TypeError("cu_seqlens must be a CUDA int32 tensor")
        return make_desc(1, Ntok, H, dk, dv, dt, mode, cu_seqlens, cu_seqlens.numel() - 1), cu_seqlens.numel() - 1
    B = B if B is not None else 1
    T = T if T is not None else Ntok // max(B, 1)
    if B * T != Ntok:
        raise ValueError("B*T must equal the number of tokens")
    return make_desc(B, T, H, dk, dv, dt, mode), B


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _mode(mode) -> int:
    return KLA_ISO if mode in ("iso", KLA_ISO) else KLA_DIAG


def plan(desc: KlaDesc) -> dict:
    """Segments per row, launches per call and tensor-core use for ``desc``."""
    seg, lau, tc = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().kla_plan(ctypes.byref(desc), ctypes.byref(seg), ctypes.byref(lau), ctypes.byref(tc)), "kla_plan")
    return {"segments": seg.value, "launches": lau.value, "tensor_core": bool(tc.value)}


def workspace_bytes(desc: KlaDesc) -> int:
    return int(lib().kla_workspace_bytes(ctypes.byref(desc)))


def forward(q, k, v, a, qn, beta, lambda0=None, eta0=None, cu_seqlens=None, B=None, T=None,
            mode="diag", final_state=False, out=None, workspace=None):
    """KLA forward on CUDA tensors in the layouts of include/kla.h.
    Returns ``out`` or ``(out, final_lambda, final_eta)`` with ``final_state``."""
    m = _mode(mode)
    desc, N = _desc_from(q, v, B, T, m, cu_seqlens)
    for name, t in (("q", q), ("k", k), ("v", v), ("a", a), ("qn", qn), ("beta", beta)):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share a dtype")
    for name, t in (("a", a), ("qn", qn), ("beta", beta), ("lambda0", lambda0), ("eta0", eta0)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32" % name)
    H, dk, dv = q.shape[1], q.shape[2], v.shape[2]
    if out is None:
        out = torch.empty(q.shape[0], H, dv, dtype=q.dtype, device=q.device)
    fl = fe = None
    if final_state:
        fl = torch.empty((N, H) if m == KLA_ISO else (N, H, dk), dtype=torch.float32, device=q.device)
        fe = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    nbytes = workspace_bytes(desc)
    if workspace is None and nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    s = lib().kla_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(qn), _ptr(beta),
                          _ptr(lambda0), _ptr(eta0), _ptr(out), _ptr(fl), _ptr(fe), _ptr(workspace),
                          nbytes, _stream())
    _check(s, "kla_forward")
    return (out, fl, fe) if final_state else out


def kdn_forward(q, k, v, a, qn, beta, lambda0=None, M0=None, cu_seqlens=None, B=None, T=None,
                mode="diag", final_state=False, out=None):
    """Kalman Delta Network forward (the Kalman-gain residual write) on CUDA
    tensors in the layouts of include/kla.h. Returns ``out`` or
    ``(out, final_lambda, final_M)`` with ``final_state`` (final_M: the
    posterior mean [N,H,dk,dv])."""
    m = _mode(mode)
    desc, N = _desc_from(q, v, B, T, m, cu_seqlens)
    for name, t in (("q", q), ("k", k), ("v", v), ("a", a), ("qn", qn), ("beta", beta)):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share a dtype")
    for name, t in (("a", a), ("qn", qn), ("beta", beta), ("lambda0", lambda0), ("M0", M0)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32" % name)
    H, dk, dv = q.shape[1], q.shape[2], v.shape[2]
    if out is None:
        out = torch.empty(q.shape[0], H, dv, dtype=q.dtype, device=q.device)
    fl = fm = None
    if final_state:
        fl = torch.empty((N, H) if m == KLA_ISO else (N, H, dk), dtype=torch.float32, device=q.device)
        fm = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    s = lib().kla_kdn_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(qn), _ptr(beta),
                              _ptr(lambda0), _ptr(M0), _ptr(out), _ptr(fl), _ptr(fm), _stream())
    _check(s, "kla_kdn_forward")
    return (out, fl, fm) if final_state else out


def backward(q, k, v, a, qn, beta, dout, lambda0=None, eta0=None, dfinal_lambda=None, dfinal_eta=None,
             cu_seqlens=None, B=None, T=None, mode="diag", workspace=None):
    """Gradients of ``forward`` (include/kla.h kla_backward) on CUDA tensors:
    returns a dict of fp32 tensors ``dq, dk, dv, da, dqn, dbeta, dlambda0,
    deta0`` in the layouts of the corresponding inputs."""
    m = _mode(mode)
    desc, N = _desc_from(q, v, B, T, m, cu_seqlens)
    for name, t in (("q", q), ("k", k), ("v", v), ("a", a), ("qn", qn), ("beta", beta), ("dout", dout)):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if k.dtype != q.dtype or v.dtype != q.dtype or dout.dtype != q.dtype:
        raise TypeError("q, k, v, dout must share a dtype")
    for name, t in (("a", a), ("qn", qn), ("beta", beta), ("lambda0", lambda0), ("eta0", eta0),
                    ("dfinal_lambda", dfinal_lambda), ("dfinal_eta", dfinal_eta)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32" % name)
    H, dk, dv = q.shape[1], q.shape[2], v.shape[2]
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32), "dv": torch.empty(v.shape, **f32),
         "da": torch.empty(a.shape, **f32), "dqn": torch.empty(qn.shape, **f32),
         "dbeta": torch.empty(beta.shape, **f32),
         "dlambda0": torch.empty((N, H) if m == KLA_ISO else (N, H, dk), **f32),
         "deta0": torch.empty(N, H, dk, dv, **f32)}
    nbytes = lib().kla_backward_workspace_bytes(ctypes.byref(desc))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    s = lib().kla_backward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(qn), _ptr(beta),
                           _ptr(lambda0), _ptr(eta0), _ptr(dout), _ptr(dfinal_lambda), _ptr(dfinal_eta),
                           *(_ptr(g[n]) for n in ("dq", "dk", "dv", "da", "dqn", "dbeta", "dlambda0", "deta0")),
                           _ptr(workspace), workspace.numel(), _stream())
    _check(s, "kla_backward")
    return g


def prologue(xq, xk, xv, xa, xqn, xbeta, wq, wk, wv, bq=None, bk=None, bv=None, cu_seqlens=None,
             B=None, T=None, mode="diag", out=None):
    """The mixer's input prologue on CUDA tensors (include/kla.h kla_prologue):
    returns ``(q, k, v, a, qn, beta)`` in the forward pass's layouts."""
    m = _mode(mode)
    desc, N = _desc_from(xq, xv, B, T, m, cu_seqlens)
    ts = (xq, xk, xv, xa, xqn, xbeta, wq, wk, wv) + tuple(t for t in (bq, bk, bv) if t is not None)
    for t in ts:
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("prologue inputs must be contiguous CUDA tensors")
    W = wq.shape[-1]
    if out is None:
        out = (torch.empty_like(xq), torch.empty_like(xk), torch.empty_like(xv), torch.empty_like(xa),
               torch.empty_like(xqn), torch.empty_like(xbeta))
    s = lib().kla_prologue(ctypes.byref(desc), W, *[_ptr(t) for t in (xq, xk, xv, xa, xqn, xbeta, wq, wk, wv,
                                                                        bq, bk, bv)],
                           *[_ptr(t) for t in out], _stream())
    _check(s, "kla_prologue")
    return out


def precision(k, a, qn, beta, lambda0=None, cu_seqlens=None, B=None, T=None, mode="diag"):
    """Posterior precision after every token ([Ntok,H,dk], iso [Ntok,H])."""
    m = _mode(mode)
    desc, N = _desc_from(k, k, B, T, m, cu_seqlens)
    Ntok, H, dk = k.shape
    lam = torch.empty((Ntok, H) if m == KLA_ISO else (Ntok, H, dk), dtype=torch.float32, device=k.device)
    nbytes = int(lib().kla_precision_workspace_bytes(ctypes.byref(desc)))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=k.device) if nbytes else None
    s = lib().kla_precision(ctypes.byref(desc), _ptr(k), _ptr(a), _ptr(qn), _ptr(beta), _ptr(lambda0),
                            _ptr(lam), _ptr(ws), nbytes, _stream())
    _check(s, "kla_precision")
    return lam


def decode_step(q, k, v, a, qn, beta, lam, eta, mode="diag", out=None):
    """One recurrent step per row: q,k,v [N,H,d], a,qn [N,H,dk] (iso [N,H]),
    beta [N,H]; ``lam``/``eta`` (the belief) are updated in place. Returns out."""
    m = _mode(mode)
    N, H, dk = q.shape
    dv = v.shape[-1]
    desc = make_desc(N, 1, H, dk, dv, KLA_BF16 if q.dtype == torch.bfloat16 else KLA_FP32, m)
    if out is None:
        out = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    s = lib().kla_decode_step(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(qn), _ptr(beta),
                              _ptr(lam), _ptr(eta), _ptr(out), _stream())
    _check(s, "kla_decode_step")
    return out


def host_device_bytes(desc: KlaDesc) -> int:
    return int(lib().kla_host_device_bytes(ctypes.byref(desc)))


def forward_host(desc: KlaDesc, q, k, v, a, qn, beta, out, lambda0=None, eta0=None,
                 final_lambda=None, final_eta=None, device_buffer=None, stream=None):
    """kla_forward_host on CPU tensors (pinned for asynchronous copies). The
    call copies inputs in, runs, copies results out and synchronises."""
    nbytes = host_device_bytes(desc)
    if device_buffer is None:
        device_buffer = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    s = lib().kla_forward_host(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(qn), _ptr(beta),
                               _ptr(lambda0), _ptr(eta0), _ptr(out), _ptr(final_lambda), _ptr(final_eta),
                               _ptr(device_buffer), nbytes, st)
    _check(s, "kla_forward_host")
    return out


def forward_noalloc(q, k, v, a, qn, beta, lambda0=None, eta0=None, B=None, T=None, mode="diag",
                    final_state=False, out=None):
    """kla_forward_noalloc: the forward pass with the library's fixed device
    scratch area as workspace, for callers that cannot allocate device memory
    (outputs passed in via ``out`` are used as given)."""
    m = _mode(mode)
    desc, N = _desc_from(q, v, B, T, m, None)
    H, dk, dv = q.shape[1], q.shape[2], v.shape[2]
    if out is None:
        out = torch.empty(q.shape[0], H, dv, dtype=q.dtype, device=q.device)
    fl = fe = None
    if final_state:
        fl = torch.empty((N, H) if m == KLA_ISO else (N, H, dk), dtype=torch.float32, device=q.device)
        fe = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    s = lib().kla_forward_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(qn), _ptr(beta),
                                  _ptr(lambda0), _ptr(eta0), _ptr(out), _ptr(fl), _ptr(fe), _stream())
    _check(s, "kla_forward_noalloc")
    return (out, fl, fe) if final_state else out


def check(stream=None):
    """Synchronise and read the device status word (raises on an error)."""
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    _check(lib().kla_check(st), "kla_check")
