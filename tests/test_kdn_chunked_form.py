"""The chunked (UT-transform) form of the Kalman Delta Network residual write,
in fp64, equals the oracle's token-by-token recursion for every chunk size.

The write is M_t = diag(a_t) M_{t-1} + gamma_t w_t r_t^T with the residual
r_t = v_t - (diag(a_t) M_{t-1})^T k_t, w_t = k_t / lambda~_t and
gamma_t = beta_t / (1 + beta_t k_t.w_t); w and gamma depend only on the
precision chain. Per chunk, with Gamma the decay product from the chunk start,
K~ = k Gamma, Q~ = q Gamma, W~ = gamma w / Gamma and M_0 the mean at the chunk
start, the residuals solve a unit lower-triangular system
    (I + strict_lower(K~ W~^T)) R = V - K~ M_0,
and then
    O = Q~ M_0 + lower(Q~ W~^T) R,      M_end = Gamma_end (M_0 + W~^T R).
These are the equations a tensor-core KDN kernel evaluates chunk by chunk; the
test fixes them against the oracle before any kernel does.
"""
import numpy as np
import pytest

import oracle


def chunked_kdn(x, T, C):
    q, k, v, a, qn, beta = (x[n] for n in ("q", "k", "v", "a", "qn", "beta"))
    _, H, dk = q.shape
    dv = v.shape[2]
    out = np.zeros((T, H, dv))
    fl, fm = np.zeros((1, H, dk)), np.zeros((1, H, dk, dv))
    for h in range(H):
        # the precision chain alone gives the write direction and gain of every token
        lam, W = x["lam0"][0, h].copy(), np.zeros((T, dk))
        for t in range(T):
            lt = lam / (a[t, h] ** 2 + qn[t, h] * lam)
            w = k[t, h] / lt
            W[t] = beta[t, h] / (1.0 + beta[t, h] * k[t, h] @ w) * w
            lam = lt + beta[t, h] * k[t, h] ** 2
        fl[0, h] = lam
        M = x["M0"][0, h].copy()
        for t0 in range(0, T, C):
            t1 = min(T, t0 + C)
            Gam = np.cumprod(a[t0:t1, h], axis=0)
            Kt, Qt, Wt = k[t0:t1, h] * Gam, q[t0:t1, h] * Gam, W[t0:t1] / Gam
            n = t1 - t0
            R = np.linalg.solve(np.eye(n) + np.tril(Kt @ Wt.T, -1), v[t0:t1, h] - Kt @ M)
            out[t0:t1, h] = Qt @ M + np.tril(Qt @ Wt.T) @ R
            M = Gam[-1][:, None] * (M + Wt.T @ R)
        fm[0, h] = M
    return {"out": out, "final_lambda": fl, "final_M": fm}


@pytest.mark.parametrize("C", [1, 5, 16, 64])
def test_kdn_chunked_form_equals_the_oracle(C):
    rng = np.random.default_rng(2)
    T, H, dk, dv = 41, 2, 8, 4
    f = lambda y: np.asarray(y, dtype=np.float32).astype(np.float64)  # noqa: E731
    kk = rng.standard_normal((T, H, dk))
    x = dict(q=f(rng.standard_normal((T, H, dk))), k=f(kk / np.linalg.norm(kk, axis=-1, keepdims=True)),
             v=f(rng.standard_normal((T, H, dv))), a=f(rng.uniform(0.6, 0.999, (T, H, dk))),
             qn=f(rng.uniform(0.0, 0.2, (T, H, dk))), beta=f(rng.uniform(0.2, 3.0, (T, H))),
             lam0=f(rng.uniform(0.5, 2.0, (1, H, dk))), M0=f(rng.standard_normal((1, H, dk, dv))))
    got = chunked_kdn(x, T, C)
    want = oracle.kdn_forward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], x["lam0"], x["M0"], B=1, T=T)
    for name in ("out", "final_lambda", "final_M"):
        err = np.max(np.abs(got[name] - want[name]) / (1.0 + np.abs(want[name])))
        assert err < 1e-9, (name, err)
