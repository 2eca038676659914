"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle (oracle/kla_oracle.c) against a statement the
mathematics or the pages fix, chosen so that a plausible slip in the oracle
(a dropped term, the gate taken from the updated precision, a readout from
the prior, a transposed index) fails at least one of them:

* a textbook covariance-form Kalman filter (predicted variance, Kalman gain,
  innovation) per key: the information form must equal the covariance form
  (Kalman Linear Attention abstract: the information-form reparameterisation
  is exact Bayesian filtering);
* a full-matrix Kalman filter with one-hot keys, where the diagonal posterior
  is exact;
* closed forms: no dynamics (a=1, qn=0) gives running precision-weighted
  means; qn=0, beta=0 gives pure decay of the mean; constant parameters drive
  lambda to the Moebius fixed point (the OU prior keeps precision bounded,
  KLA technical summary, ablation remark);
* a two-step example worked by hand in exact fractions (tests/golden);
* invariants: associativity of the Moebius composition under every grouping
  (KLA technical summary section 2), determinant, positivity, split-call
  equivalence of the state hand-off, varlen = separate calls, head
  equivariance, thread-count invariance.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs, random_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(rng, Ntok, H, dk, dv, iso=False, zero_keys=False):
    q = rng.standard_normal((Ntok, H, dk)).astype(np.float32)
    k = rng.standard_normal((Ntok, H, dk)).astype(np.float32)
    if zero_keys:
        k[rng.random((Ntok, H, dk)) < 0.2] = 0.0
    v = rng.standard_normal((Ntok, H, dv)).astype(np.float32)
    shp = (Ntok, H) if iso else (Ntok, H, dk)
    a = (0.3 + 0.9 * rng.random(shp)).astype(np.float32)         # a in (0.3, 1.2)
    qn = (0.5 * rng.random(shp)).astype(np.float32)
    beta = (0.1 + 2.0 * rng.random((Ntok, H))).astype(np.float32)
    return q, k, v, a, qn, beta


def covariance_form_kf(q, k, v, a, qn, beta, lam0, eta0, B, T):
    """Textbook scalar Kalman filter per key i, written in covariance form.

    State: row m_i in R^dv with variance P_i. Transition m <- a m, P <- a^2 P + qn.
    Observation of the token: v = k_i m_i + noise of precision beta, i.e.
    y = v / k_i with noise variance R = 1/(beta k_i^2). Standard gain update.
    Readout: o = sum_i q_i m_i (posterior mean through the query)."""
    Ntok, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((Ntok, H, dv))
    lam_traj = np.zeros((Ntok, H, dk))
    fl = np.zeros((B, H, dk))
    fe = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            P = 1.0 / lam0[b, h].astype(np.float64)
            m = eta0[b, h].astype(np.float64) * P[:, None]
            for t in range(b * T, (b + 1) * T):
                at = a[t, h].astype(np.float64)
                Pbar = at * at * P + qn[t, h]
                mbar = at[:, None] * m
                for i in range(dk):
                    ki = float(k[t, h, i])
                    if ki == 0.0:
                        P[i], m[i] = Pbar[i], mbar[i]
                        continue
                    R = 1.0 / (float(beta[t, h]) * ki * ki)
                    K = Pbar[i] / (Pbar[i] + R)
                    y = v[t, h].astype(np.float64) / ki
                    m[i] = mbar[i] + K * (y - mbar[i])
                    P[i] = (1.0 - K) * Pbar[i]
                out[t, h] = q[t, h].astype(np.float64) @ m
                lam_traj[t, h] = 1.0 / P
            fl[b, h] = 1.0 / P
            fe[b, h] = m / P[:, None]
    return out, lam_traj, fl, fe


def assert_close(x, y, rtol=1e-10, atol=1e-12):
    np.testing.assert_allclose(x, y, rtol=rtol, atol=atol)


# --------------------------------------------------------------------------

def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_t2.json")))
    x = g["inputs"]
    one = lambda key: np.array(x[key], np.float32).reshape(2, 1, 1)
    r = oracle.forward(one("q"), one("k"), one("v"), one("a"), one("qn"),
                       np.array(x["beta"], np.float32).reshape(2, 1), B=1, T=2)
    e = g["expected"]
    want = [Fraction(n, d) for n, d in zip(e["out_num"], e["out_den"])]
    assert_close(r["out"].ravel(), [float(f) for f in want], rtol=1e-14)
    assert r["final_lambda"].item() == pytest.approx(17 / 12, rel=1e-14)
    assert r["final_eta"].item() == pytest.approx(3 / 2, rel=1e-14)


@pytest.mark.parametrize("zero_keys", [False, True])
def test_information_form_equals_covariance_form(zero_keys):
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 2, 40, 2, 4, 3
    q, k, v, a, qn, beta = rand_case(rng, B * T, H, dk, dv, zero_keys=zero_keys)
    lam0 = (0.5 + rng.random((B, H, dk))).astype(np.float32)
    eta0 = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    r = oracle.forward(q, k, v, a, qn, beta, lam0, eta0, B=B, T=T, want_lambda=True)
    out, lt, fl, fe = covariance_form_kf(q, k, v, a, qn, beta, lam0, eta0, B, T)
    assert_close(r["out"], out, rtol=1e-9, atol=1e-11)
    assert_close(r["lambda"], lt)
    assert_close(r["final_lambda"], fl)
    assert_close(r["final_eta"], fe, rtol=1e-9, atol=1e-11)


def test_one_hot_keys_equal_full_matrix_kalman_filter():
    """With one-hot keys the full-covariance posterior stays diagonal, so the
    diagonal information filter is exact; compare to a dense matrix KF."""
    rng = np.random.default_rng(5)
    T, H, dk, dv = 30, 1, 5, 3
    q, _, v, a, qn, beta = rand_case(rng, T, H, dk, dv)
    k = np.zeros((T, H, dk), np.float32)
    idx = rng.integers(0, dk, T)
    scale = (0.5 + rng.random(T)).astype(np.float32)
    k[np.arange(T), 0, idx] = scale
    lam0 = (0.5 + rng.random((1, H, dk))).astype(np.float32)
    eta0 = rng.standard_normal((1, H, dk, dv)).astype(np.float32)
    r = oracle.forward(q, k, v, a, qn, beta, lam0, eta0, B=1, T=T)

    Sig = np.diag(1.0 / lam0[0, 0].astype(np.float64))
    X = Sig @ eta0[0, 0].astype(np.float64)
    outs = []
    for t in range(T):
        A = np.diag(a[t, 0].astype(np.float64))
        Sig = A @ Sig @ A + np.diag(qn[t, 0].astype(np.float64))
        X = A @ X
        kt = k[t, 0].astype(np.float64)
        S = kt @ Sig @ kt + 1.0 / float(beta[t, 0])
        K = Sig @ kt / S
        X = X + np.outer(K, v[t, 0].astype(np.float64) - kt @ X)
        Sig = Sig - np.outer(K, kt @ Sig)
        outs.append(q[t, 0].astype(np.float64) @ X)
    assert_close(r["out"][:, 0], np.array(outs), rtol=1e-9, atol=1e-11)
    Lam = np.linalg.inv(Sig)
    assert_close(r["final_lambda"][0, 0], np.diag(Lam), rtol=1e-9)
    assert_close(r["final_eta"][0, 0], Lam @ X, rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("iso", [False, True])
def test_no_dynamics_gives_running_precision_weighted_mean(iso):
    rng = np.random.default_rng(3)
    T, H, dk, dv = 50, 2, 4, 3
    q, k, v, _, _, beta = rand_case(rng, T, H, dk, dv)
    shp = (T, H) if iso else (T, H, dk)
    a = np.ones(shp, np.float32)
    qn = np.zeros(shp, np.float32)
    r = oracle.forward(q, k, v, a, qn, beta, B=1, T=T, iso=iso, want_lambda=True)
    k64, v64, b64 = k.astype(np.float64), v.astype(np.float64), beta.astype(np.float64)
    if iso:
        lam = 1.0 + np.cumsum(b64 * (k64 ** 2).sum(-1) / dk, axis=0)          # [T,H]
        lam_k = lam[:, :, None]
    else:
        lam = 1.0 + np.cumsum(b64[:, :, None] * k64 ** 2, axis=0)             # [T,H,dk]
        lam_k = lam
    eta = np.cumsum(b64[:, :, None, None] * k64[:, :, :, None] * v64[:, :, None, :], axis=0)
    out = np.einsum("thi,thij->thj", q.astype(np.float64) / lam_k, eta)
    assert_close(r["lambda"], lam)
    assert_close(r["out"], out, rtol=1e-9, atol=1e-11)


def test_pure_decay_of_the_mean():
    rng = np.random.default_rng(4)
    T, H, dk, dv = 25, 2, 3, 2
    q, k, v, a, _, _ = rand_case(rng, T, H, dk, dv)
    qn = np.zeros_like(a)
    beta = np.zeros((T, H), np.float32)
    lam0 = (0.5 + rng.random((1, H, dk))).astype(np.float32)
    m0 = rng.standard_normal((1, H, dk, dv))
    eta0 = (m0 * lam0[..., None]).astype(np.float32)
    r = oracle.forward(q, k, v, a, qn, beta, lam0, eta0, B=1, T=T, want_lambda=True)
    m0 = eta0.astype(np.float64) / lam0.astype(np.float64)[..., None]
    prod_a = np.cumprod(a.astype(np.float64), axis=0)                          # [T,H,dk]
    assert_close(r["lambda"], lam0.astype(np.float64) / prod_a ** 2)
    want = np.einsum("thi,hij->thj", q.astype(np.float64) * prod_a, m0[0])
    assert_close(r["out"], want, rtol=1e-9, atol=1e-12)


def test_constant_parameters_reach_moebius_fixed_point():
    T, H, dk, dv = 4000, 1, 3, 1
    a_c = np.array([0.95, 0.7, 1.0])
    qn_c = np.array([0.05, 0.3, 0.01])
    b_c = np.array([0.5, 0.1, 0.02])
    a = np.tile(a_c, (T, H, 1)).astype(np.float32)
    qn = np.tile(qn_c, (T, H, 1)).astype(np.float32)
    k = np.tile(np.sqrt(b_c), (T, H, 1)).astype(np.float32)
    beta = np.ones((T, H), np.float32)
    q = np.ones((T, H, dk), np.float32)
    v = np.ones((T, H, dv), np.float32)
    r = oracle.forward(q, k, v, a, qn, beta, B=1, T=T, want_lambda=True)
    a64, qn64 = a[0, 0].astype(np.float64), qn[0, 0].astype(np.float64)
    b64 = k[0, 0].astype(np.float64) ** 2
    # lambda* is the positive root of qn x^2 + (a^2 - 1 - b qn) x - b a^2 = 0
    A_, B_, C_ = qn64, a64 ** 2 - 1 - b64 * qn64, -b64 * a64 ** 2
    root = (-B_ + np.sqrt(B_ ** 2 - 4 * A_ * C_)) / (2 * A_)
    assert_close(r["lambda"][-1, 0], root, rtol=1e-9)
    assert np.all(r["lambda"] > 0)


def test_moebius_element_is_one_filter_step_and_composition_is_associative():
    rng = np.random.default_rng(7)
    T = 7
    a = 0.3 + 0.9 * rng.random(T)
    qn = 0.5 * rng.random(T)
    kk = rng.standard_normal(T)
    beta = 0.1 + 2 * rng.random(T)
    lam0 = float(np.float32(0.8))  # the oracle reads fp32 inputs
    r = oracle.forward(np.ones((T, 1, 1), np.float32), kk.astype(np.float32).reshape(T, 1, 1),
                       np.ones((T, 1, 1), np.float32), a.astype(np.float32).reshape(T, 1, 1),
                       qn.astype(np.float32).reshape(T, 1, 1), beta.astype(np.float32).reshape(T, 1),
                       np.array([[[lam0]]], np.float32), B=1, T=T, want_lambda=True)
    a32, qn32 = a.astype(np.float32).astype(np.float64), qn.astype(np.float32).astype(np.float64)
    b = beta.astype(np.float32).astype(np.float64) * kk.astype(np.float32).astype(np.float64) ** 2
    Ms = [oracle.mobius_element(a32[t], qn32[t], b[t]) for t in range(T)]
    for t in range(T):
        assert np.linalg.det(Ms[t].reshape(2, 2)) == pytest.approx(a32[t] ** 2, rel=1e-12)

    def groupings(lo, hi):
        # every binary bracketing of M_hi ... M_lo (later maps on the left)
        if lo == hi:
            yield Ms[lo]
            return
        for s in range(lo, hi):
            for left in groupings(s + 1, hi):
                for right in groupings(lo, s):
                    yield oracle.mobius_compose(left, right)

    for t in range(T):
        seen = 0
        for M in groupings(0, t):
            assert oracle.mobius_apply(M, lam0) == pytest.approx(r["lambda"][t, 0, 0], rel=1e-12)
            # projective: any positive rescaling is the same map
            assert oracle.mobius_apply(M / M.max(), lam0) == pytest.approx(r["lambda"][t, 0, 0], rel=1e-12)
            seen += 1
        catalan = [1, 1, 2, 5, 14, 42, 132][t]
        assert seen == catalan
    P = Ms[0]
    for t in range(1, T):
        P = oracle.mobius_compose(Ms[t], P)
    assert np.linalg.det(P.reshape(2, 2)) == pytest.approx(np.prod(a32 ** 2), rel=1e-10)


@pytest.mark.parametrize("iso", [False, True])
def test_split_call_equals_one_call(iso):
    rng = np.random.default_rng(9)
    T, T1, H, dk, dv = 60, 23, 2, 4, 3
    q, k, v, a, qn, beta = rand_case(rng, T, H, dk, dv, iso=iso)
    full = oracle.forward(q, k, v, a, qn, beta, B=1, T=T, iso=iso)
    p1 = oracle.forward(q[:T1], k[:T1], v[:T1], a[:T1], qn[:T1], beta[:T1], B=1, T=T1, iso=iso)
    p2 = oracle.forward(q[T1:], k[T1:], v[T1:], a[T1:], qn[T1:], beta[T1:],
                        p1["final_lambda"].astype(np.float32), p1["final_eta"].astype(np.float32),
                        B=1, T=T - T1, iso=iso)
    # the hand-off state is rounded to fp32 (the interface's state dtype)
    assert_close(np.concatenate([p1["out"], p2["out"]]), full["out"], rtol=1e-5, atol=1e-6)
    assert_close(p2["final_lambda"], full["final_lambda"], rtol=1e-6)
    assert_close(p2["final_eta"], full["final_eta"], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("iso", [False, True])
def test_varlen_equals_separate_calls_and_heads_are_independent(iso):
    rng = np.random.default_rng(13)
    lens = [5, 17, 1, 30]
    Ntok, H, dk, dv = sum(lens), 3, 4, 2
    q, k, v, a, qn, beta = rand_case(rng, Ntok, H, dk, dv, iso=iso)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N = len(lens)
    lam0 = (0.5 + rng.random((N, H) if iso else (N, H, dk))).astype(np.float32)
    eta0 = rng.standard_normal((N, H, dk, dv)).astype(np.float32)
    r = oracle.forward(q, k, v, a, qn, beta, lam0, eta0, cu_seqlens=cu, iso=iso)
    for n in range(N):
        s, e = cu[n], cu[n + 1]
        rn = oracle.forward(q[s:e], k[s:e], v[s:e], a[s:e], qn[s:e], beta[s:e],
                            lam0[n:n + 1], eta0[n:n + 1], B=1, T=e - s, iso=iso)
        np.testing.assert_array_equal(r["out"][s:e], rn["out"])
        np.testing.assert_array_equal(r["final_lambda"][n], rn["final_lambda"][0])
        np.testing.assert_array_equal(r["final_eta"][n], rn["final_eta"][0])
    perm = np.array([2, 0, 1])
    rp = oracle.forward(q[:, perm], k[:, perm], v[:, perm], a[:, perm], qn[:, perm], beta[:, perm],
                        lam0[:, perm], eta0[:, perm], cu_seqlens=cu, iso=iso)
    np.testing.assert_array_equal(rp["out"], r["out"][:, perm])


def test_isotropic_with_one_key_equals_diagonal():
    rng = np.random.default_rng(17)
    T, H, dv = 40, 2, 3
    q, k, v, a, qn, beta = rand_case(rng, T, H, 1, dv)
    rd = oracle.forward(q, k, v, a, qn, beta, B=1, T=T)
    ri = oracle.forward(q, k, v, a[..., 0], qn[..., 0], beta, B=1, T=T, iso=True)
    assert_close(ri["out"], rd["out"], rtol=1e-14)
    assert_close(ri["final_lambda"], rd["final_lambda"][..., 0], rtol=1e-14)


def test_thread_count_does_not_change_results():
    w = WORKLOADS[1].with_(T=64, B=2)
    inp = make_inputs(w)
    r1 = oracle.forward_inputs(inp, w, num_threads=1)
    r4 = oracle.forward_inputs(inp, w, num_threads=4)
    for key in r1:
        np.testing.assert_array_equal(r1[key], r4[key])


@pytest.mark.parametrize("wid", [0, 1, 4])
def test_workload_precisions_stay_positive_and_bounded(wid):
    w = WORKLOADS[wid]
    if wid == 1:
        w = w.with_(T=256)
    if wid == 4:
        w = w.with_(T=2048, H=4, len_lo=64, len_hi=1024)
    inp = make_inputs(w)
    r = oracle.forward_inputs(inp, w, want_lambda=True)
    lam = r["lambda"]
    assert np.all(lam > 0) and np.all(np.isfinite(lam))
    assert np.all(np.isfinite(r["out"]))


def test_unit_subrange_matches_full_run():
    w = WORKLOADS[1].with_(T=32)
    inp = make_inputs(w)
    full = oracle.forward_inputs(inp, w, want_final=False)
    part = oracle.forward_inputs(inp, w, want_final=False, units=(5, 9))
    H = w.H
    for u in range(5, 9):
        n, h = divmod(u, H)
        np.testing.assert_array_equal(part["out"][n * w.T:(n + 1) * w.T, h],
                                      full["out"][n * w.T:(n + 1) * w.T, h])
