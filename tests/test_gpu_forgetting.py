"""Strong forgetting inside a chunk, on the GPU against the oracle.

The forget gate g = a/(a^2 + qn*lambda) (Kalman Linear Attention, technical
summary section 3: forget gates come from precision ratios) can fall far
below one when the OU decay a is small or the process noise qn*lambda is
large (the OU prior of technical summary section 1 allows both). The chunk
kernel then meets log2-gate ranges inside one 64-token chunk that a single
reference per key cannot span; it takes such chunks in two or four passes
with their own references. These tests drive that region and check every
output against the oracle at the bf16 tolerance, with the library status
KLA_OK. The last test reaches the one residual limit (a 16-token block whose
log2-gate range exceeds what one reference represents) and checks that
kla_check reports KLA_ERR_RANGE instead of returning silently.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs, random_state
from test_gpu_parity import ERRORS, TOL, close, run  # noqa: F401

pytestmark = pytest.mark.gpu


def check_against_oracle(w, inp, lam0=None, eta0=None):
    out, fl, fe = run(w, inp, lam0, eta0)
    x = dict(inp)
    x["lambda0"], x["eta0"] = lam0, eta0
    ref = oracle.forward_inputs(x, w)
    tol = TOL[w.dtype]
    close(out, ref["out"], tol, "out")
    close(fl, ref["final_lambda"], tol, "final_lambda")
    close(fe, ref["final_eta"], tol, "final_eta")


def log2_gate_span(inp, w, ref_lambda, width=64):
    """Largest per-key range of the cumulative log2 gate over one aligned
    window of `width` tokens (a chunk, half a chunk or a quarter), from the
    oracle's precision trajectory: shows which pass level the inputs reach."""
    a = inp["a"].double().numpy()
    qn = inp["qn"].double().numpy()
    lam = ref_lambda
    prev = np.concatenate([np.ones_like(lam[:1]), lam[:-1]], axis=0)
    G = np.log2(a / (a * a + qn * prev))
    T = G.shape[0] // w.B
    worst = 0.0
    for b in range(w.B):
        Gb = G[b * T:(b + 1) * T]
        for c0 in range(0, T - width + 1, width):
            cs = np.cumsum(Gb[c0:c0 + width], axis=0)
            worst = max(worst, float((cs.max(axis=0) - np.minimum(cs.min(axis=0), 0)).max()))
    return worst


def spans(inp, w):
    ref = oracle.forward_inputs(inp, w, want_lambda=True, want_out=False, want_final=False)
    return [log2_gate_span(inp, w, ref["lambda"], width) for width in (64, 32, 16)]


@pytest.mark.parametrize("segments", ["1", "3"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("a_mu,qn_mu", [(-1.0, 0.0), (-2.0, 0.5)])
def test_strong_forgetting_diag(monkeypatch, d, segments, a_mu, qn_mu):
    # a = sigmoid(N(-1, 1)) (median 0.27), qn = softplus(N(0, 1)): about -2 log2 per
    # token; a = sigmoid(N(-2, 1)) (median 0.12): every chunk spans more than one
    # reference in some key and takes two passes
    monkeypatch.setenv("KLA_SEGMENTS", segments)
    w = WORKLOADS[2].with_(B=2, H=2, T=1000, dk=d, dv=d, a_mu=a_mu, qn_mu=qn_mu)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=40 + d)
    s64, s32, s16 = spans(inp, w)
    assert s16 <= 160 and (a_mu > -2 or s64 > 160)
    check_against_oracle(w, inp, lam0, eta0)


@pytest.mark.parametrize("segments", ["1", "4"])
def test_forget_burst_after_calm_stretch(monkeypatch, segments):
    # calm gates (a ~ 0.95), then bursts of strong forgetting inside chunks
    monkeypatch.setenv("KLA_SEGMENTS", segments)
    w = WORKLOADS[2].with_(B=1, H=3, T=1600, dk=128, dv=128)
    inp = make_inputs(w)
    a, qn = inp["a"], inp["qn"]
    a[300:360] = 0.01
    qn[300:360] = 1.0
    a[700:716, 1] = 0.02          # one head, one 16-token quarter
    qn[700:716, 1] = 4.0
    a[1101:1150, :, :64] = 0.05   # half of the keys, across a chunk boundary
    qn[1101:1150, :, :64] = 2.0
    s64, s32, s16 = spans(inp, w)
    assert s32 > 160 >= s16      # some chunks take four passes of 16 tokens
    check_against_oracle(w, inp)


@pytest.mark.parametrize("segments", ["1", "3"])
def test_isotropic_strong_forgetting(monkeypatch, segments):
    # one precision per head, a = sigmoid(N(-0.85, 1)) (median 0.3), qn = softplus(N(0, 1))
    monkeypatch.setenv("KLA_SEGMENTS", segments)
    w = WORKLOADS[4].with_(B=2, H=3, T=1200, varlen=False, iso_sigmoid=True, a_mu=-0.85, qn_mu=0.0,
                           final_state=True)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=9)
    check_against_oracle(w, inp, lam0, eta0)


def test_isotropic_strong_forgetting_packed():
    w = WORKLOADS[4].with_(B=2, H=2, T=1500, len_lo=1, len_hi=500, iso_sigmoid=True, a_mu=-0.85, qn_mu=0.0)
    check_against_oracle(w, make_inputs(w))


def test_range_limit_is_reported():
    # 32 tokens of one key with a gate near 2^-20 (a = 0.01, qn = 1e6): a 16-token
    # quarter spans ~300 in log2, beyond one reference; the call reports it
    w = WORKLOADS[2].with_(B=1, H=2, T=256, dk=128, dv=128)
    inp = make_inputs(w)
    inp["a"][96:128, 0, 5] = 0.01
    inp["qn"][96:128, 0, 5] = 1e6
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=w.B, T=w.T)
    with pytest.raises(kla.KlaError) as e:
        kla.check()
    assert e.value.status == kla.KLA_ERR_RANGE
    # the status word is cleared by the check: a valid call afterwards is clean
    w2 = WORKLOADS[2].with_(B=1, H=2, T=256)
    check_against_oracle(w2, make_inputs(w2))


def test_bounded_wait_reports_timeout(monkeypatch):
    # With the tile loads withheld (a test switch of the library), the gate's
    # first wait on them never completes: after the bounded wait the kernel sets
    # the abort flag, every role leaves through its teardown, and the status word
    # reports KLA_ERR_TIMEOUT. No fault, no hang: the context stays usable and a
    # valid call afterwards is clean.
    w = WORKLOADS[1].with_(B=1, H=2, T=200)
    inp = make_inputs(w)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    # whole rows (one launch: the walk kernel alone meets the withheld tiles)
    monkeypatch.setenv("KLA_SEGMENTS", "1")
    monkeypatch.setenv("KLA_TEST_WITHHOLD_TILES", "1")
    kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=w.B, T=w.T)
    with pytest.raises(kla.KlaError) as e:
        kla.check()
    assert e.value.status == kla.KLA_ERR_TIMEOUT
    monkeypatch.delenv("KLA_TEST_WITHHOLD_TILES")
    monkeypatch.delenv("KLA_SEGMENTS")
    check_against_oracle(w, inp)
