"""GPU parity of the KLA gradients (kla_backward) against the fp64 oracle's
reverse mode (oracle.backward, itself pinned by finite differences) on the
same seeded inputs.

Bar, per element of every gradient:
    |gpu - oracle| <= tol * (scale + |oracle|),  scale = max |oracle| of that gradient,
with tol = 2e-3: the kernels compute in fp32 from the same (bf16 or fp32)
input values the oracle reads, so the difference is fp32 rounding, summed
over the sequence in the adjoint recursions.
"""
import numpy as np
import pytest
import torch

import oracle
from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs, random_state

pytestmark = pytest.mark.gpu

TOL = 2e-3
NAMES = ("dq", "dk", "dv", "da", "dqn", "dbeta", "dlambda0", "deta0")


def grads_close(got, want, label, units=None, H=None, bounds=None):
    for name in NAMES:
        g = got[name].detach().cpu().double().numpy()
        w = want[name]
        if units is not None:
            idx = []
            for u in range(*units):
                n, h = divmod(u, H)
                if name in ("dlambda0", "deta0"):
                    idx.append((g[n, h], w[n, h]))
                else:
                    s, e = bounds(n)
                    idx.append((g[s:e, h], w[s:e, h]))
            g = np.concatenate([x[0].ravel() for x in idx])
            w = np.concatenate([x[1].ravel() for x in idx])
        scale = float(np.max(np.abs(w))) if w.size else 0.0
        err = float(np.max(np.abs(g - w) / (scale + np.abs(w) + 1e-30))) if w.size else 0.0
        print("%-40s %-9s %.3e  (tol %.0e)" % (label, name, err, TOL))
        assert err <= TOL, (label, name, err)


def run(w, inp, lam0=None, eta0=None, dfl=None, dfe=None, seed=0, units=None):
    g = torch.Generator().manual_seed(seed + 101)
    dout = torch.randn(inp["v"].shape, generator=g).to(inp["v"].dtype)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    c = lambda t: t.cuda() if t is not None else None  # noqa: E731
    got = kla.backward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], dout.cuda(), c(lam0), c(eta0), c(dfl),
                       c(dfe), cu_seqlens=d["cu_seqlens"], B=w.B, T=w.T, mode=w.mode)
    torch.cuda.synchronize()
    kla.check()
    want = oracle.backward(inp["q"], inp["k"], inp["v"], inp["a"], inp["qn"], inp["beta"], dout, lam0, eta0,
                           dfl, dfe, cu_seqlens=inp["cu_seqlens"],
                           B=None if inp["cu_seqlens"] is not None else w.B,
                           T=None if inp["cu_seqlens"] is not None else w.T, iso=w.mode == "iso", units=units)
    return got, want


def state_grads(w, N, seed):
    g = torch.Generator().manual_seed(seed + 7)
    nl = (N, w.H) if w.mode == "iso" else (N, w.H, w.dk)
    return torch.randn(nl, generator=g), torch.randn(N, w.H, w.dk, w.dv, generator=g)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["diag", "iso"])
def test_backward_head_dims(dk, dv, dtype, mode):
    base = WORKLOADS[4] if mode == "iso" else WORKLOADS[2]
    w = base.with_(B=2, H=2, T=120, dk=dk, dv=dv, dtype=dtype, varlen=False)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=dk + dv)
    dfl, dfe = state_grads(w, w.B, dk + dv)
    got, want = run(w, inp, lam0.float(), eta0.float(), dfl, dfe, seed=dk)
    grads_close(got, want, "bwd %s %s %dx%d" % (mode, dtype, dk, dv))


@pytest.mark.parametrize("T", [1, 2, 65, 300])
def test_backward_lengths_and_default_state(T):
    w = WORKLOADS[1].with_(B=2, H=3, T=T)
    got, want = run(w, make_inputs(w), seed=T)
    grads_close(got, want, "bwd T=%d" % T)


@pytest.mark.parametrize("mode", ["diag", "iso"])
def test_backward_packed_sequences(mode):
    base = WORKLOADS[4] if mode == "iso" else WORKLOADS[1]
    w = base.with_(B=1, H=2, T=900, varlen=True, len_lo=1, len_hi=200, dk=64, dv=64)
    inp = make_inputs(w)
    N = inp["cu_seqlens"].numel() - 1
    lam0, eta0 = random_state(w, N, seed=3)
    dfl, dfe = state_grads(w, N, 3)
    got, want = run(w, inp, lam0.float(), eta0.float(), dfl, dfe, seed=3)
    grads_close(got, want, "bwd packed %s" % mode)


def test_backward_empty_input():
    w = WORKLOADS[1].with_(B=2, H=2, T=0)
    inp = make_inputs(w)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    got = kla.backward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], torch.empty_like(d["v"]), B=w.B, T=0)
    assert got["dq"].numel() == 0


def test_backward_layer_workload_sampled_units():
    # the 1.3B-layer shape (B=8, H=16, T=4096, d=128); the oracle checks two units
    w = WORKLOADS[2]
    inp = make_inputs(w)
    got, want = run(w, inp, seed=11, units=(0, 2))
    grads_close(got, want, "bwd 1.3B layer", units=(0, 2), H=w.H,
                bounds=lambda n: (n * w.T, (n + 1) * w.T))
