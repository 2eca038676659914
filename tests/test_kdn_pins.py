"""Pins of the Kalman Delta Network oracle (the Kalman-gain residual write).

The pages (Kalman Delta Networks abstract) state the method without equations:
the memory is the state of a linear-Gaussian model, the Kalman gain weights each
residual write, diagonal KDN projects each one-step posterior onto diagonal
Gaussians, and the delta rule is the special case of a token-wise isotropic
surrogate for the predictive covariance without covariance tracking. Each pin
below checks the oracle against something fixed outside it: a dense textbook
Kalman update, the scalar Kalman filter, the (separately pinned) KLA filter on
one-hot keys, and a plain gated delta rule.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(rng, *shape, lo=None, hi=None):
    if lo is not None:
        return rng.uniform(lo, hi, size=shape).astype(np.float32)
    return rng.standard_normal(shape).astype(np.float32)


def _one_step_inputs(rng, dk, dv, iso):
    q = _rand(rng, 1, 1, dk)
    k = _rand(rng, 1, 1, dk)
    v = _rand(rng, 1, 1, dv)
    a = _rand(rng, 1, 1, lo=0.5, hi=1.0) if iso else _rand(rng, 1, 1, dk, lo=0.5, hi=1.0)
    qn = _rand(rng, 1, 1, lo=0.05, hi=0.5) if iso else _rand(rng, 1, 1, dk, lo=0.05, hi=0.5)
    beta = _rand(rng, 1, 1, lo=0.5, hi=3.0)
    lam0 = _rand(rng, 1, 1, lo=0.5, hi=4.0) if iso else _rand(rng, 1, 1, dk, lo=0.5, hi=4.0)
    M0 = _rand(rng, 1, 1, dk, dv)
    return q, k, v, a, qn, beta, lam0, M0


@pytest.mark.parametrize("iso", [False, True])
def test_one_step_is_the_dense_kalman_update(iso):
    # From a diagonal (isotropic) prior, one KDN step is the textbook Kalman
    # update with the full covariance: same posterior mean; the precision is the
    # diagonal of the posterior precision matrix (iso: its mean diagonal).
    rng = np.random.default_rng(3 + iso)
    dk, dv = 5, 3
    q, k, v, a, qn, beta, lam0, M0 = _one_step_inputs(rng, dk, dv, iso)
    res = oracle.kdn_forward(q, k, v, a, qn, beta, lam0, M0, B=1, T=1, iso=iso)
    kk = k[0, 0].astype(np.float64)
    av = np.full(dk, float(a[0, 0])) if iso else a[0, 0].astype(np.float64)
    qv = np.full(dk, float(qn[0, 0])) if iso else qn[0, 0].astype(np.float64)
    l0 = np.full(dk, float(lam0[0, 0])) if iso else lam0[0, 0].astype(np.float64)
    b = float(beta[0, 0])
    P0 = np.diag(1.0 / l0)
    A = np.diag(av)
    Mp = A @ M0[0, 0].astype(np.float64)                   # predicted mean
    Pp = A @ P0 @ A.T + np.diag(qv)                          # predicted covariance
    S = kk @ Pp @ kk + 1.0 / b                               # innovation variance
    K = Pp @ kk / S                                          # Kalman gain
    M1 = Mp + np.outer(K, v[0, 0] - kk @ Mp)                 # posterior mean
    P1 = Pp - np.outer(K, kk) @ Pp                           # posterior covariance
    prec = np.linalg.inv(P1)
    np.testing.assert_allclose(res["final_M"][0, 0], M1, rtol=1e-10, atol=1e-12)
    want_lam = np.mean(np.diag(prec)) if iso else np.diag(prec)
    np.testing.assert_allclose(res["final_lambda"][0, 0], want_lam, rtol=1e-10)
    np.testing.assert_allclose(res["out"][0, 0], M1.T @ q[0, 0].astype(np.float64), rtol=1e-10, atol=1e-12)


def test_scalar_key_is_the_kalman_filter():
    # dk = 1: the diagonal is the whole covariance, so every step is exact; the
    # covariance-form scalar Kalman filter over many steps, per value column.
    rng = np.random.default_rng(11)
    T, dv = 40, 4
    q = _rand(rng, T, 1, 1)
    k = _rand(rng, T, 1, 1)
    v = _rand(rng, T, 1, dv)
    a = _rand(rng, T, 1, 1, lo=0.3, hi=1.2)
    qn = _rand(rng, T, 1, 1, lo=0.0, hi=0.7)
    beta = _rand(rng, T, 1, lo=0.1, hi=5.0)
    lam0 = np.array([[[2.0]]], dtype=np.float32)
    M0 = _rand(rng, 1, 1, 1, dv)
    res = oracle.kdn_forward(q, k, v, a, qn, beta, lam0, M0, B=1, T=T)
    m = M0[0, 0, 0].astype(np.float64)
    p = 1.0 / 2.0
    for t in range(T):
        at, qt, kt, bt = float(a[t, 0, 0]), float(qn[t, 0, 0]), float(k[t, 0, 0]), float(beta[t, 0])
        m = at * m
        p = at * at * p + qt
        gain = p * kt / (kt * kt * p + 1.0 / bt)
        m = m + gain * (v[t, 0].astype(np.float64) - kt * m)
        p = p - gain * kt * p
        np.testing.assert_allclose(res["out"][t, 0], float(q[t, 0, 0]) * m, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(res["final_M"][0, 0, 0], m, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(res["final_lambda"][0, 0, 0], 1.0 / p, rtol=1e-9)


def test_one_hot_keys_coincide_with_the_kla_filter():
    # One-hot keys decouple the keys: the KDN write and the KLA filter's
    # information-form update give the same posterior mean (M = eta / lambda).
    rng = np.random.default_rng(5)
    T, dk, dv = 50, 6, 4
    idx = rng.integers(0, dk, size=T)
    k = np.zeros((T, 1, dk), np.float32)
    k[np.arange(T), 0, idx] = rng.choice([-1.5, 0.7, 1.0, 2.0], size=T)
    q = _rand(rng, T, 1, dk)
    v = _rand(rng, T, 1, dv)
    a = _rand(rng, T, 1, dk, lo=0.6, hi=1.0)
    qn = _rand(rng, T, 1, dk, lo=0.0, hi=0.3)
    beta = _rand(rng, T, 1, lo=0.2, hi=3.0)
    lam0 = _rand(rng, 1, 1, dk, lo=0.5, hi=2.0)
    M0 = _rand(rng, 1, 1, dk, dv)
    kdn = oracle.kdn_forward(q, k, v, a, qn, beta, lam0, M0, B=1, T=T)
    eta0 = (M0.astype(np.float64) * lam0[..., None].astype(np.float64)).astype(np.float32)
    # eta0 rounded to fp32 for the KLA oracle's input: compare at fp32 accuracy
    kla = oracle.forward(q, k, v, a, qn, beta, lam0, eta0, B=1, T=T)
    np.testing.assert_allclose(kdn["out"], kla["out"], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(kdn["final_lambda"], kla["final_lambda"], rtol=1e-12)
    np.testing.assert_allclose(kdn["final_M"], kla["final_eta"] / kla["final_lambda"][..., None],
                               rtol=1e-5, atol=1e-6)


def test_constant_isotropic_surrogate_is_the_gated_delta_rule():
    # Choose qn per token so that the isotropic predictive precision is a
    # constant c (no covariance tracking in effect): the KDN write becomes the
    # gated delta rule M = a (I - b' k k^T) M + b' k v^T with b' = beta/(c + beta)
    # for unit keys.
    rng = np.random.default_rng(9)
    T, dk, dv, c = 60, 8, 5, 1.7
    k = _rand(rng, T, 1, dk)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = _rand(rng, T, 1, dk)
    v = _rand(rng, T, 1, dv)
    a = _rand(rng, T, 1, lo=0.8, hi=1.0)
    beta = _rand(rng, T, 1, lo=0.3, hi=2.0)
    lam = 2.5
    qn = np.zeros((T, 1), np.float32)
    for t in range(T):
        at = float(a[t, 0])
        qn[t, 0] = (lam / c - at * at) / lam          # lambda~ = lam / (a^2 + qn lam) = c
        ksq = float(np.dot(k[t, 0].astype(np.float64), k[t, 0].astype(np.float64)))
        lam = c + float(beta[t, 0]) * ksq / dk
    res = oracle.kdn_forward(q, k, v, a, qn, beta, np.array([[2.5]], np.float32), None, B=1, T=T, iso=True)
    M = np.zeros((dk, dv))
    for t in range(T):
        kt = k[t, 0].astype(np.float64)
        bp = float(beta[t, 0]) / (c + float(beta[t, 0]) * np.dot(kt, kt))
        M = float(a[t, 0]) * M
        M = M + bp * np.outer(kt, v[t, 0] - kt @ M)
        np.testing.assert_allclose(res["out"][t, 0], M.T @ q[t, 0].astype(np.float64), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("iso", [False, True])
def test_split_call_and_packed_sequences(iso):
    rng = np.random.default_rng(21 + iso)
    T, H, dk, dv = 37, 2, 4, 3
    q = _rand(rng, T, H, dk)
    k = _rand(rng, T, H, dk)
    v = _rand(rng, T, H, dv)
    a = _rand(rng, T, H, lo=0.7, hi=1.0) if iso else _rand(rng, T, H, dk, lo=0.7, hi=1.0)
    qn = _rand(rng, T, H, lo=0.0, hi=0.2) if iso else _rand(rng, T, H, dk, lo=0.0, hi=0.2)
    beta = _rand(rng, T, H, lo=0.2, hi=2.0)
    whole = oracle.kdn_forward(q, k, v, a, qn, beta, B=1, T=T, iso=iso)
    t1 = 15
    first = oracle.kdn_forward(q[:t1], k[:t1], v[:t1], a[:t1], qn[:t1], beta[:t1], B=1, T=t1, iso=iso)
    second = oracle.kdn_forward(q[t1:], k[t1:], v[t1:], a[t1:], qn[t1:], beta[t1:],
                                first["final_lambda"].astype(np.float32), first["final_M"].astype(np.float32),
                                B=1, T=T - t1, iso=iso)
    np.testing.assert_allclose(np.concatenate([first["out"], second["out"]]), whole["out"], rtol=1e-5, atol=1e-6)
    # packed: two sequences equal two separate calls
    cu = np.array([0, t1, T], np.int32)
    packed = oracle.kdn_forward(q, k, v, a, qn, beta, cu_seqlens=cu, iso=iso)
    np.testing.assert_allclose(packed["out"][:t1], first["out"], rtol=1e-12, atol=1e-14)
    alone = oracle.kdn_forward(q[t1:], k[t1:], v[t1:], a[t1:], qn[t1:], beta[t1:], B=1, T=T - t1, iso=iso)
    np.testing.assert_allclose(packed["out"][t1:], alone["out"], rtol=1e-12, atol=1e-14)
