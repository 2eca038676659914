"""CPU oracle for the Kalman linear-attention forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use this package; the product path
(``bayesian_filter_scan_b200``) never imports it, and this package never
imports the product path. The arithmetic lives in ``kla_oracle.c`` (plain C,
fp64, the sequential filter written out step by step); this module compiles it
with gcc and marshals numpy / torch CPU arrays through ctypes.

Parity status: pinned. The tests check the oracle against a textbook
covariance-form Kalman filter, a full-matrix Kalman filter on one-hot keys,
closed forms, a hand-worked example and invariants (see tests/test_oracle_pins.py).
The Kalman Delta Network residual write (``kdn_forward``) is pinned against the
textbook dense Kalman update for one step from a diagonal prior, the scalar
Kalman filter for dk = 1, the KLA filter on one-hot keys, and the gated delta
rule when the predictive covariance is a constant isotropic surrogate (see
tests/test_kdn_pins.py). The mixer's input prologue (``prologue``: causal conv,
SiLU, L2 norm, sigmoid / softplus gates) is plain numpy, pinned against the
identity kernel, numpy's convolution per channel, closed forms of the gates
and packed sequences (tests/test_prologue_pins.py). The gradients of the filter
(``backward``, reverse mode over stored states) are pinned against central
finite differences of the pinned forward (tests/test_backward_pins.py).
The isotropic increment beta*|k|^2/dk is pinned for consistency only (it
reduces to the diagonal filter when dk = 1 and to the closed form when a=1,
qn=0); the choice of that constant is a reading of the Kalman Delta Networks
abstract, which gives no equation for it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kla_oracle.c")
_LIB = os.path.join(_HERE, "libkla_oracle.so")
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libkla_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.kla_oracle_forward.restype = ctypes.c_int
        lib.kla_oracle_forward.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, ctypes.c_int,
            _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p,
            _f64p, _f64p, _f64p, _f64p, ctypes.c_long, ctypes.c_long, ctypes.c_int]
        lib.kdn_oracle_forward.restype = ctypes.c_int
        lib.kdn_oracle_forward.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, ctypes.c_int,
            _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p,
            _f64p, _f64p, _f64p, ctypes.c_long, ctypes.c_long, ctypes.c_int]
        lib.kla_oracle_backward.restype = ctypes.c_int
        lib.kla_oracle_backward.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, ctypes.c_int,
            _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p,
            _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p,
            ctypes.c_long, ctypes.c_long, ctypes.c_int]
        lib.kla_oracle_max_threads.restype = ctypes.c_int
        lib.kla_oracle_mobius_element.argtypes = [ctypes.c_double] * 3 + [_f64p]
        lib.kla_oracle_mobius_compose.argtypes = [_f64p, _f64p, _f64p]
        lib.kla_oracle_mobius_apply.argtypes = [_f64p, ctypes.c_double]
        lib.kla_oracle_mobius_apply.restype = ctypes.c_double
        _lib = lib
    return _lib


def _f32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (bf16 upcasts exactly to fp32)
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(arr, typ):
    return None if arr is None else arr.ctypes.data_as(typ)


def max_threads() -> int:
    return int(_load().kla_oracle_max_threads())


def forward(q, k, v, a, qn, beta, lambda0=None, eta0=None, cu_seqlens=None,
            B=None, T=None, iso=False, want_out=True, want_final=True,
            want_lambda=False, units=None, num_threads=0):
    """Run the sequential filter. Arrays use the layouts of the CUDA path
    (tokens flattened over the batch). Returns a dict of float64 numpy arrays:
    ``out`` [Ntok,H,dv], ``final_lambda`` [N,H,dk] (iso [N,H]), ``final_eta``
    [N,H,dk,dv] and, if asked, ``lambda`` (posterior precision after every
    token). ``units=(begin, end)`` restricts the work to units n*H+h in
    [begin, end) (other entries are left zero)."""
    lib = _load()
    q, k, v, a, qn, beta = (_f32(x) for x in (q, k, v, a, qn, beta))
    lambda0, eta0 = _f32(lambda0), _f32(eta0)
    Ntok, H, dk = q.shape
    dv = v.shape[-1]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        N = cu.size - 1
        B_, T_ = 1, Ntok
    else:
        B_ = B if B is not None else 1
        T_ = T if T is not None else Ntok // B_
        assert B_ * T_ == Ntok
        N = B_
    res = {}
    out = np.zeros((Ntok, H, dv)) if want_out else None
    fl = np.zeros((N, H) if iso else (N, H, dk)) if want_final else None
    fe = np.zeros((N, H, dk, dv)) if want_final else None
    lt = np.zeros((Ntok, H) if iso else (Ntok, H, dk)) if want_lambda else None
    ub, ue = (0, -1) if units is None else units
    err = lib.kla_oracle_forward(
        B_, T_, H, dk, dv, int(bool(iso)), _ptr(cu, _i32p), N,
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(a, _f32p), _ptr(qn, _f32p),
        _ptr(beta, _f32p), _ptr(lambda0, _f32p), _ptr(eta0, _f32p),
        _ptr(out, _f64p), _ptr(fl, _f64p), _ptr(fe, _f64p), _ptr(lt, _f64p),
        int(ub), int(ue), int(num_threads))
    if err:
        raise RuntimeError("oracle failed (bad shape or out of memory)")
    if want_out:
        res["out"] = out
    if want_final:
        res["final_lambda"], res["final_eta"] = fl, fe
    if want_lambda:
        res["lambda"] = lt
    return res


def backward(q, k, v, a, qn, beta, dout, lambda0=None, eta0=None, dfinal_lambda=None,
             dfinal_eta=None, cu_seqlens=None, B=None, T=None, iso=False, units=None, num_threads=0):
    """Gradients of ``forward`` (reverse mode over the stored per-token states,
    kla_oracle.c): given dout [Ntok,H,dv] and optionally the gradients of the
    final state, returns float64 arrays ``dq, dk, dv, da, dqn, dbeta`` (the
    shapes of the inputs), ``dlambda0`` [N,H,dk] (iso [N,H]) and ``deta0``
    [N,H,dk,dv]. ``units`` restricts the work as in ``forward``."""
    lib = _load()
    q, k, v, a, qn, beta, dout = (_f32(x) for x in (q, k, v, a, qn, beta, dout))
    lambda0, eta0, dfl, dfe = (_f32(x) for x in (lambda0, eta0, dfinal_lambda, dfinal_eta))
    Ntok, H, dk = q.shape
    dv = v.shape[-1]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        N = cu.size - 1
        B_, T_ = 1, Ntok
    else:
        B_ = B if B is not None else 1
        T_ = T if T is not None else Ntok // B_
        assert B_ * T_ == Ntok
        N = B_
    g = {"dq": np.zeros(q.shape), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape),
         "da": np.zeros(a.shape), "dqn": np.zeros(qn.shape), "dbeta": np.zeros(beta.shape),
         "dlambda0": np.zeros((N, H) if iso else (N, H, dk)), "deta0": np.zeros((N, H, dk, dv))}
    ub, ue = (0, -1) if units is None else units
    err = lib.kla_oracle_backward(
        B_, T_, H, dk, dv, int(bool(iso)), _ptr(cu, _i32p), N,
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(a, _f32p), _ptr(qn, _f32p),
        _ptr(beta, _f32p), _ptr(lambda0, _f32p), _ptr(eta0, _f32p), _ptr(dout, _f32p),
        _ptr(dfl, _f32p), _ptr(dfe, _f32p),
        *(_ptr(g[n], _f64p) for n in ("dq", "dk", "dv", "da", "dqn", "dbeta", "dlambda0", "deta0")),
        int(ub), int(ue), int(num_threads))
    if err:
        raise RuntimeError("oracle backward failed (bad shape or out of memory)")
    return g


def kdn_forward(q, k, v, a, qn, beta, lambda0=None, M0=None, cu_seqlens=None,
                B=None, T=None, iso=False, units=None, num_threads=0):
    """Kalman Delta Network forward with the Kalman-gain residual write (the
    reading in kla_oracle.c: the exact Kalman mean update from a diagonal /
    isotropic prior, the posterior precision projected back onto it). Returns
    ``out`` [Ntok,H,dv], ``final_lambda`` [N,H,dk] (iso [N,H]) and ``final_M``
    [N,H,dk,dv] (the posterior mean), float64."""
    lib = _load()
    q, k, v, a, qn, beta = (_f32(x) for x in (q, k, v, a, qn, beta))
    lambda0, M0 = _f32(lambda0), _f32(M0)
    Ntok, H, dk = q.shape
    dv = v.shape[-1]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        N = cu.size - 1
        B_, T_ = 1, Ntok
    else:
        B_ = B if B is not None else 1
        T_ = T if T is not None else Ntok // B_
        assert B_ * T_ == Ntok
        N = B_
    out = np.zeros((Ntok, H, dv))
    fl = np.zeros((N, H) if iso else (N, H, dk))
    fm = np.zeros((N, H, dk, dv))
    ub, ue = (0, -1) if units is None else units
    err = lib.kdn_oracle_forward(
        B_, T_, H, dk, dv, int(bool(iso)), _ptr(cu, _i32p), N,
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(a, _f32p), _ptr(qn, _f32p),
        _ptr(beta, _f32p), _ptr(lambda0, _f32p), _ptr(M0, _f32p),
        _ptr(out, _f64p), _ptr(fl, _f64p), _ptr(fm, _f64p), int(ub), int(ue), int(num_threads))
    if err:
        raise RuntimeError("oracle failed (bad shape or out of memory)")
    return {"out": out, "final_lambda": fl, "final_M": fm}


def kdn_forward_inputs(inp: dict, w, **kw):
    """``kdn_forward`` on a dict produced by the seeded input generator."""
    return kdn_forward(inp["q"], inp["k"], inp["v"], inp["a"], inp["qn"], inp["beta"],
                       inp.get("lambda0"), inp.get("M0"), inp.get("cu_seqlens"),
                       B=None if inp.get("cu_seqlens") is not None else w.B,
                       T=None if inp.get("cu_seqlens") is not None else w.T,
                       iso=(w.mode == "iso"), **kw)


def forward_inputs(inp: dict, w, **kw):
    """``forward`` on a dict produced by the seeded input generator."""
    return forward(inp["q"], inp["k"], inp["v"], inp["a"], inp["qn"], inp["beta"],
                   inp.get("lambda0"), inp.get("eta0"), inp.get("cu_seqlens"),
                   B=None if inp.get("cu_seqlens") is not None else w.B,
                   T=None if inp.get("cu_seqlens") is not None else w.T,
                   iso=(w.mode == "iso"), **kw)


# ---- Moebius helpers (2x2 matrix form of one predict+update step) ----------

def mobius_element(a: float, qn: float, b: float) -> np.ndarray:
    M = np.zeros(4)
    _load().kla_oracle_mobius_element(a, qn, b, _ptr(M, _f64p))
    return M


def mobius_compose(L: np.ndarray, R: np.ndarray) -> np.ndarray:
    out = np.zeros(4)
    L = np.ascontiguousarray(L, dtype=np.float64)
    R = np.ascontiguousarray(R, dtype=np.float64)
    _load().kla_oracle_mobius_compose(_ptr(L, _f64p), _ptr(R, _f64p), _ptr(out, _f64p))
    return out


def mobius_apply(M: np.ndarray, lam: float) -> float:
    M = np.ascontiguousarray(M, dtype=np.float64)
    return float(_load().kla_oracle_mobius_apply(_ptr(M, _f64p), float(lam)))


def time_forward(inp: dict, w, units, num_threads=0) -> tuple:
    """Wall-clock seconds of the oracle on a sub-range of units (CPU baseline)."""
    t0 = time.perf_counter()
    forward_inputs(inp, w, units=units, want_final=False, num_threads=num_threads)
    return time.perf_counter() - t0


# ---- fused prologue of the mixer (1-D causal conv + SiLU, L2 norm, gates) ---

PROLOGUE_EPS = 1e-6


def prologue(xq, xk, xv, xa, xqn, xbeta, wq, wk, wv, bq=None, bk=None, bv=None, cu_seqlens=None,
             B=None, T=None):
    """The mixer's input prologue (Kalman Linear Attention, technical summary
    section 4: a Mamba-like block with a 1-D causal convolution and SiLU), in
    plain numpy fp64, step by step:
      q = l2norm(silu(conv(xq))), k = l2norm(silu(conv(xk))), v = silu(conv(xv)),
      a = sigmoid(xa), qn = softplus(xqn), beta = sigmoid(xbeta),
    conv: per channel c of head h, y[t] = b[h,c] + sum_{w<W} wgt[h,c,w] x[t-(W-1)+w]
    with x = 0 before the start of t's sequence (each packed sequence starts
    afresh); l2norm over dk: y / sqrt(sum y^2 + PROLOGUE_EPS). Layouts as the
    forward's inputs: x* [Ntok,H,d] (xa, xqn [Ntok,H,dk] or [Ntok,H]),
    weights [H,d,W], biases [H,d]. Returns float64 arrays."""
    def f64(x):
        if x is None:
            return None
        if hasattr(x, "detach"):
            x = x.detach().cpu().double().numpy()
        return np.asarray(x, dtype=np.float64)
    xq, xk, xv, xa, xqn, xbeta = (f64(x) for x in (xq, xk, xv, xa, xqn, xbeta))
    wq, wk, wv, bq, bk, bv = (f64(x) for x in (wq, wk, wv, bq, bk, bv))
    Ntok = xq.shape[0]
    if cu_seqlens is not None:
        cu = np.asarray(cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
    else:
        B_ = B if B is not None else 1
        T_ = T if T is not None else Ntok // B_
        cu = np.arange(B_ + 1, dtype=np.int64) * T_

    def conv(x, wgt, bias):
        Wd = wgt.shape[-1]
        y = np.zeros_like(x)
        for n in range(cu.size - 1):
            s, e = int(cu[n]), int(cu[n + 1])
            for t in range(s, e):
                acc = np.zeros(x.shape[1:]) if bias is None else bias.copy()
                for w in range(Wd):
                    src = t - (Wd - 1) + w
                    if src >= s:
                        acc = acc + wgt[..., w] * x[src]
                y[t] = acc
        return y

    def silu(y):
        return y / (1.0 + np.exp(-y))

    def l2norm(y):
        return y / np.sqrt(np.sum(y * y, axis=-1, keepdims=True) + PROLOGUE_EPS)

    def sigmoid(y):
        return 1.0 / (1.0 + np.exp(-y))

    def softplus(y):
        return np.log1p(np.exp(-np.abs(y))) + np.maximum(y, 0.0)

    return {"q": l2norm(silu(conv(xq, wq, bq))), "k": l2norm(silu(conv(xk, wk, bk))),
            "v": silu(conv(xv, wv, bv)), "a": sigmoid(xa), "qn": softplus(xqn), "beta": sigmoid(xbeta)}
