"""GPU parity of the Kalman Delta Network residual write (kla_kdn_forward)
against the fp64 oracle (oracle.kdn_forward) on the same seeded inputs.

Bar, per element of out / final_lambda / final_M:
    |gpu - oracle| <= tol * (1 + |oracle|)
with tol = 2e-2 for bf16 inputs (bf16 outputs) and 1e-4 for fp32 inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs, random_state

from test_gpu_parity import close

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def run_kdn(w, inp, lam0=None, M0=None):
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    r = kla.kdn_forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"],
                        lam0.cuda() if lam0 is not None else None, M0.cuda() if M0 is not None else None,
                        cu_seqlens=d["cu_seqlens"], B=w.B, T=w.T, mode=w.mode, final_state=True)
    torch.cuda.synchronize()
    kla.check()
    return r


def compare(w, inp, lam0=None, M0=None, units=None):
    out, fl, fm = run_kdn(w, inp, lam0, M0)
    x = dict(inp)
    x["lambda0"], x["M0"] = lam0, M0
    ref = oracle.kdn_forward_inputs(x, w, units=units)
    tol = TOL[w.dtype]
    if units is None:
        close(out, ref["out"], tol, "kdn out")
        close(fl, ref["final_lambda"], tol, "kdn final_lambda")
        close(fm, ref["final_M"], tol, "kdn final_M")
    else:
        for u in range(*units):
            n, h = divmod(u, w.H)
            s, e = n * w.T, (n + 1) * w.T
            close(out[s:e, h], ref["out"][s:e, h], tol, "kdn out unit %d" % u)
            close(fl[n, h], ref["final_lambda"][n, h], tol, "kdn final_lambda unit %d" % u)
            close(fm[n, h], ref["final_M"][n, h], tol, "kdn final_M unit %d" % u)


def prior(w, N, seed):
    lam0, eta0 = random_state(w, N, seed=seed)
    # a prior mean of a moderate size (eta0 / lambda0 of the generator's belief)
    M0 = (eta0 / (lam0[..., None] if w.mode == "diag" else lam0[..., None, None])).float()
    return lam0, M0.contiguous()


@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 128), (32, 64), (64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["diag", "iso"])
def test_kdn_head_dims(dk, dv, dtype, mode):
    base = WORKLOADS[4] if mode == "iso" else WORKLOADS[2]
    w = base.with_(B=2, H=2, T=150, dk=dk, dv=dv, dtype=dtype, varlen=False)
    inp = make_inputs(w)
    lam0, M0 = prior(w, w.B, seed=dk + dv)
    compare(w, inp, lam0, M0)


@pytest.mark.parametrize("T", [0, 1, 7, 64, 333])
def test_kdn_ragged_lengths(T):
    w = WORKLOADS[1].with_(B=2, H=3, T=T)
    inp = make_inputs(w)
    if T == 0:
        d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        out = kla.kdn_forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=w.B, T=0)
        assert out.numel() == 0
        return
    compare(w, inp)


@pytest.mark.parametrize("mode", ["diag", "iso"])
def test_kdn_packed_sequences(mode):
    base = WORKLOADS[4] if mode == "iso" else WORKLOADS[1]
    w = base.with_(B=2, H=2, T=1200, varlen=True, len_lo=1, len_hi=500, dk=64, dv=64)
    inp = make_inputs(w)
    N = inp["cu_seqlens"].numel() - 1
    lam0, M0 = prior(w, N, seed=4)
    compare(w, inp, lam0, M0)


def test_kdn_one_hot_keys_match_the_kla_path():
    # With one-hot keys the residual write and the KLA filter coincide (a pinned
    # property of the oracles); the two CUDA paths must agree as well.
    w = WORKLOADS[1].with_(B=1, H=2, T=300, dk=64, dv=64, dtype="fp32")
    inp = make_inputs(w)
    g = torch.Generator().manual_seed(17)
    idx = torch.randint(0, w.dk, (w.T * w.B, w.H), generator=g)
    k = torch.zeros_like(inp["k"])
    k.scatter_(2, idx[..., None], 1.0)
    inp["k"] = k
    d = {kk: (v.cuda() if v is not None else None) for kk, v in inp.items()}
    kdn = kla.kdn_forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=w.B, T=w.T)
    kl = kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=w.B, T=w.T)
    torch.cuda.synchronize()
    close(kdn, kl.cpu().double().numpy(), 1e-4, "kdn vs kla, one-hot keys")


def test_kdn_layer_workload_sampled_units():
    # the 1.3B-layer shape (B=8, H=16, T=4096, d=128) in the launch the bench times;
    # the oracle checks two (row, head) units
    w = WORKLOADS[2]
    compare(w, make_inputs(w), units=(0, 2))
