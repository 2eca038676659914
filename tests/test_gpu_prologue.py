"""GPU parity of the mixer's input prologue (kla_prologue: causal conv + SiLU,
L2 norm, gate activations) against the numpy oracle (oracle.prologue).

Bar, per element: |gpu - oracle| <= tol * (1 + |oracle|), tol = 2e-2 for bf16
outputs (q, k, v; the fp32 gates use 1e-4) and 1e-4 for fp32 inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs

from test_gpu_parity import close

pytestmark = pytest.mark.gpu


def pre_activations(w, seed, W=4, bias=True):
    """Synthetic pre-activations and conv weights of a workload's shape."""
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    inp = make_inputs(w)                      # for the token count and packed offsets
    Ntok, H, dk, dv = inp["q"].shape[0], w.H, w.dk, w.dv
    nl = dk if w.mode == "diag" else None
    r = lambda *s: torch.randn(*s, generator=g)  # noqa: E731
    x = {
        "xq": r(Ntok, H, dk).to(dt), "xk": r(Ntok, H, dk).to(dt), "xv": r(Ntok, H, dv).to(dt),
        "xa": (r(Ntok, H, nl) if nl else r(Ntok, H)) + 2.0, "xqn": (r(Ntok, H, nl) if nl else r(Ntok, H)) - 2.0,
        "xbeta": r(Ntok, H),
        "wq": r(H, dk, W) / W ** 0.5, "wk": r(H, dk, W) / W ** 0.5, "wv": r(H, dv, W) / W ** 0.5,
        "bq": r(H, dk) * 0.1 if bias else None, "bk": r(H, dk) * 0.1 if bias else None,
        "bv": r(H, dv) * 0.1 if bias else None,
    }
    return x, inp["cu_seqlens"]


def check(w, W=4, bias=True, seed=0):
    x, cu = pre_activations(w, seed, W, bias)
    d = {k: (v.cuda().contiguous() if v is not None else None) for k, v in x.items()}
    got = kla.prologue(**d, cu_seqlens=cu.cuda() if cu is not None else None,
                       B=None if cu is not None else w.B, T=None if cu is not None else w.T, mode=w.mode)
    torch.cuda.synchronize()
    want = oracle.prologue(**x, cu_seqlens=cu, B=None if cu is not None else w.B, T=None if cu is not None else w.T)
    tol_x = 2e-2 if w.dtype == "bf16" else 1e-4
    for name, t, tol in zip(("q", "k", "v", "a", "qn", "beta"), got, (tol_x, tol_x, tol_x, 1e-4, 1e-4, 1e-4)):
        close(t, want[name], tol, "prologue " + name)
    return got


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 128), (128, 128), (128, 256)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["diag", "iso"])
def test_prologue_dims(dk, dv, dtype, mode):
    base = WORKLOADS[4] if mode == "iso" else WORKLOADS[2]
    w = base.with_(B=2, H=3, T=70, dk=dk, dv=dv, dtype=dtype, varlen=False)
    check(w, seed=dk + dv)


@pytest.mark.parametrize("W", [1, 2, 4])
@pytest.mark.parametrize("bias", [False, True])
def test_prologue_conv_widths(W, bias):
    w = WORKLOADS[1].with_(B=2, H=2, T=45)
    check(w, W=W, bias=bias, seed=W)


def test_prologue_packed_sequences_restart_the_conv():
    w = WORKLOADS[4].with_(B=1, H=2, T=900, varlen=True, len_lo=1, len_hi=200, dk=64, dv=64)
    check(w, seed=5)


def test_prologue_feeds_the_forward():
    # the prologue's outputs are the forward's inputs, in its layouts
    w = WORKLOADS[1].with_(B=2, H=2, T=300)
    q, k, v, a, qn, beta = check(w, seed=9)
    out = kla.forward(q, k, v, a, qn, beta, B=w.B, T=w.T)
    torch.cuda.synchronize()
    kla.check()
    ref = oracle.forward(q.cpu(), k.cpu(), v.cpu(), a.cpu(), qn.cpu(), beta.cpu(), B=w.B, T=w.T)
    close(out, ref["out"], 2e-2, "forward on the prologue's outputs")
