"""The chunked (dual) form of the KLA gradients, in fp64, equals the oracle's
reverse mode for every chunk size.

Per chunk, with Gamma the gate product from the chunk start, Q' = q^ Gamma,
K' = k^ / Gamma, eta_s the state at the chunk start and D the adjoint of the
state at the chunk end (walked in reverse):
    P = mask(dO V^T),  S = mask(Q' K'^T)
    dq^ = (dO eta_s^T + P K') Gamma,  dk^ = (P^T Q') / Gamma + (V D^T) Gamma_end / Gamma
    dv  = S^T dO + (K' Gamma_end) D,  D <- Q'^T dO + Gamma_end D
then the gate term g dL/dg by its identity and the precision chain in reverse.
These are the equations a tensor-core backward evaluates chunk by chunk; the
test fixes them against the oracle before any kernel does.
"""
import numpy as np
import pytest

import oracle


def chunked_gradients(x, T, C):
    q, k, v, a, qn, beta, dout = (x[n] for n in ("q", "k", "v", "a", "qn", "beta", "dout"))
    lam0, eta0, dfl, dfe = x["lam0"], x["eta0"], x["dfl"], x["dfe"]
    _, H, dk = q.shape
    res = {n: np.zeros(x[n].shape) for n in ("q", "k", "v", "a", "qn", "beta")}
    res = {"d" + n: g for n, g in res.items()}
    res["dlambda0"], res["deta0"] = np.zeros(lam0.shape), np.zeros(eta0.shape)
    for h in range(H):
        lam, L, g = lam0[0, h].copy(), np.zeros((T, dk)), np.zeros((T, dk))
        for t in range(T):
            den = a[t, h] ** 2 + qn[t, h] * lam
            g[t] = a[t, h] / den
            lam = lam / den + beta[t, h] * k[t, h] ** 2
            L[t] = lam
        qh, kh, V, dO = q[:, h] / L, beta[:, h, None] * k[:, h], v[:, h], dout[:, h]
        chunks = [(c, min(T, c + C)) for c in range(0, T, C)]
        starts, eta = [], eta0[0, h].copy()
        for t0, t1 in chunks:
            starts.append(eta.copy())
            for t in range(t0, t1):
                eta = g[t][:, None] * eta + np.outer(kh[t], V[t])
        dqh, dkh, D = np.zeros((T, dk)), np.zeros((T, dk)), dfe[0, h].copy()
        for (t0, t1), eta_s in reversed(list(zip(chunks, starts))):
            Gam = np.cumprod(g[t0:t1], axis=0)
            Gend = Gam[-1]
            Qp, Kp = qh[t0:t1] * Gam, kh[t0:t1] / Gam
            mask = np.tril(np.ones((t1 - t0, t1 - t0)))
            S, P = (Qp @ Kp.T) * mask, (dO[t0:t1] @ V[t0:t1].T) * mask
            dqh[t0:t1] = (dO[t0:t1] @ eta_s.T + P @ Kp) * Gam
            dkh[t0:t1] = (P.T @ Qp + (V[t0:t1] @ D.T) * Gend) / Gam
            res["dv"][t0:t1, h] = S.T @ dO[t0:t1] + (Kp * Gend) @ D
            D = Qp.T @ dO[t0:t1] + Gend[:, None] * D
        res["deta0"][0, h] = D
        G, Gs = np.sum(dfe[0, h] * eta, axis=1), np.zeros((T, dk))
        for t in reversed(range(T)):
            G = G + qh[t] * dqh[t] - kh[t] * dkh[t]
            Gs[t] = G
        dl = dfl[0, h].copy()
        for t in reversed(range(T)):
            lp = L[t - 1] if t > 0 else lam0[0, h]
            dlt = dl - dqh[t] * q[t, h] / L[t] ** 2
            den = a[t, h] ** 2 + qn[t, h] * lp
            dg = Gs[t] * den / a[t, h]
            dden = -(dlt * lp + dg * a[t, h]) / den ** 2
            res["da"][t, h], res["dqn"][t, h] = dg / den + 2 * a[t, h] * dden, lp * dden
            dl = dlt / den + qn[t, h] * dden
            res["dq"][t, h] = dqh[t] / L[t]
            res["dk"][t, h] = beta[t, h] * dkh[t] + 2 * beta[t, h] * k[t, h] * dlt
            res["dbeta"][t, h] = np.sum(k[t, h] * (dkh[t] + k[t, h] * dlt))
        res["dlambda0"][0, h] = dl
    return res


@pytest.mark.parametrize("C", [1, 8, 16, 64])
def test_chunked_form_equals_the_oracles_reverse_mode(C):
    rng = np.random.default_rng(1)
    T, H, dk, dv = 37, 2, 8, 4
    f = lambda y: np.asarray(y, dtype=np.float32).astype(np.float64)  # noqa: E731
    x = dict(q=f(rng.standard_normal((T, H, dk))), k=f(rng.standard_normal((T, H, dk)) * 0.5),
             v=f(rng.standard_normal((T, H, dv))), a=f(rng.uniform(0.3, 0.99, (T, H, dk))),
             qn=f(rng.uniform(0.0, 0.5, (T, H, dk))), beta=f(rng.uniform(0.2, 3.0, (T, H))),
             dout=f(rng.standard_normal((T, H, dv))), lam0=f(rng.uniform(0.5, 2.0, (1, H, dk))),
             eta0=f(rng.standard_normal((1, H, dk, dv))), dfl=f(rng.standard_normal((1, H, dk))),
             dfe=f(rng.standard_normal((1, H, dk, dv))))
    got = chunked_gradients(x, T, C)
    want = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], x["dout"], x["lam0"], x["eta0"],
                           x["dfl"], x["dfe"], B=1, T=T)
    for name, w in want.items():
        err = np.max(np.abs(got[name] - w) / (1.0 + np.abs(w)))
        assert err < 1e-10, (name, err)
