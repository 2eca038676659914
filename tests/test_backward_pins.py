"""Pins of the oracle's gradients (oracle.backward) against central finite
differences of the oracle's forward pass, which is pinned on its own
(tests/test_oracle_pins.py).

The loss is L = <dout, out> + <dfinal_lambda, final_lambda> + <dfinal_eta,
final_eta>. Inputs are multiples of 2^-12 and the steps are 2^-12 and 2^-13, so x +- h
is exact in fp32 (the forward's input type) and the difference quotients are
taken on exactly the perturbed inputs; the forward runs in fp64, and the two
quotients are combined by Richardson extrapolation, so the remaining error is
the O(h^4) truncation, far below the tolerance.
"""
import numpy as np
import pytest

import oracle

H_STEP = 2.0 ** -12


def _q(x):
    return (np.round(np.asarray(x, dtype=np.float64) / H_STEP) * H_STEP).astype(np.float32)


def problem(seed, iso, B=2, T=5, H=2, dk=3, dv=2, strong=False, varlen=False):
    rng = np.random.default_rng(seed)
    Ntok = B * T
    nl = () if iso else (dk,)
    a_lo, a_hi = (0.02, 0.1) if strong else (0.3, 0.95)
    x = {
        "q": _q(rng.standard_normal((Ntok, H, dk))), "k": _q(rng.standard_normal((Ntok, H, dk)) * 0.7),
        "v": _q(rng.standard_normal((Ntok, H, dv))),
        "a": _q(rng.uniform(a_lo, a_hi, (Ntok, H) + nl)), "qn": _q(rng.uniform(0.05, 0.5, (Ntok, H) + nl)),
        "beta": _q(rng.uniform(0.2, 2.0, (Ntok, H))),
    }
    cu = np.array([0, 3, 4, Ntok], dtype=np.int32) if varlen else None
    N = 3 if varlen else B
    x["lambda0"] = _q(rng.uniform(0.5, 2.0, (N, H) + nl))
    x["eta0"] = _q(rng.standard_normal((N, H, dk, dv)))
    seeds = {
        "dout": rng.standard_normal((Ntok, H, dv)), "dfinal_lambda": rng.standard_normal((N, H) + nl),
        "dfinal_eta": rng.standard_normal((N, H, dk, dv)),
    }
    return x, {k_: _q(v_) for k_, v_ in seeds.items()}, cu, (None if varlen else B), (None if varlen else T)


def loss(x, d, cu, B, T, iso):
    r = oracle.forward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], x["lambda0"], x["eta0"],
                       cu_seqlens=cu, B=B, T=T, iso=iso)
    return (np.sum(d["dout"].astype(np.float64) * r["out"])
            + np.sum(d["dfinal_lambda"].astype(np.float64) * r["final_lambda"])
            + np.sum(d["dfinal_eta"].astype(np.float64) * r["final_eta"]))


def finite_difference(x, d, cu, B, T, iso, name):
    """Central differences with steps h and h/2, combined by Richardson
    extrapolation (truncation O(h^4)): strong forgetting makes the loss
    strongly curved in a and qn."""
    g = np.zeros(x[name].shape)
    flat = x[name].reshape(-1)

    def central(e, h):
        keep = flat[e]
        flat[e] = keep + np.float32(h)
        lp = loss(x, d, cu, B, T, iso)
        flat[e] = keep - np.float32(h)
        lm = loss(x, d, cu, B, T, iso)
        flat[e] = keep
        return (lp - lm) / (2 * h)
    for e in range(flat.size):
        g.reshape(-1)[e] = (4 * central(e, H_STEP / 2) - central(e, H_STEP)) / 3
    return g


NAMES = ("q", "k", "v", "a", "qn", "beta", "lambda0", "eta0")


@pytest.mark.parametrize("iso", [False, True])
@pytest.mark.parametrize("case", ["plain", "strong-forgetting", "packed"])
def test_gradients_equal_finite_differences(iso, case):
    x, d, cu, B, T = problem(3 if iso else 4, iso, strong=case == "strong-forgetting", varlen=case == "packed")
    got = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], d["dout"], x["lambda0"],
                          x["eta0"], d["dfinal_lambda"], d["dfinal_eta"], cu_seqlens=cu, B=B, T=T, iso=iso)
    for name in NAMES:
        want = finite_difference(x, d, cu, B, T, iso, name)
        have = got["d" + name]
        assert have.shape == want.shape, name
        err = np.max(np.abs(have - want) / (1.0 + np.abs(want)))
        assert err < 1e-5, (name, err)


def test_no_final_state_gradient_and_default_prior():
    # dfinal_* omitted = zero; lambda0 / eta0 omitted = 1 / 0 (their gradients still reported)
    x, d, cu, B, T = problem(9, False)
    d["dfinal_lambda"][:] = 0
    d["dfinal_eta"][:] = 0
    x["lambda0"][:] = 1
    x["eta0"][:] = 0
    full = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], d["dout"], x["lambda0"],
                           x["eta0"], d["dfinal_lambda"], d["dfinal_eta"], B=B, T=T)
    bare = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], d["dout"], B=B, T=T)
    for name in ("dq", "dk", "dv", "da", "dqn", "dbeta", "dlambda0", "deta0"):
        assert np.array_equal(full[name], bare[name]), name
