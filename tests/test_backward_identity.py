"""The backward kernels' algorithm, modelled in numpy fp64, equals the oracle's
direct reverse mode.

The CUDA backward (kla_backward) stores no per-token state: it takes the gate's
gradient from the identity
    g_t dL/dg_t = <dfinal_eta, eta_T> + sum_{tau >= t} (q^_tau dq^_tau - k^_tau dk^_tau)
(per key; q^ = q / lambda, k^ = beta k), where dq^ = eta do comes from a forward
sweep and dk^ = d v from a reverse sweep of the adjoint d_t = g_{t+1} d_{t+1} +
q^_t do_t^T. This test runs those sweeps in fp64 (the same order and formulas
as the kernels, none of their code) and checks that they reproduce the oracle's
gradients to rounding, so the kernels' parity tests measure only fp32 rounding.
"""
import numpy as np
import pytest

import oracle


def sweeps(q, k, v, a, qn, beta, dout, lam0, eta0, dfl, dfe, iso):
    Ntok, H, dk = q.shape
    dv = v.shape[2]
    B = lam0.shape[0]
    T = Ntok // B
    nl = 1 if iso else dk
    res = {n: np.zeros(x.shape) for n, x in (("dq", q), ("dk", k), ("dv", v), ("da", a), ("dqn", qn),
                                              ("dbeta", beta))}
    res["dlambda0"] = np.zeros(lam0.shape)
    res["deta0"] = np.zeros(eta0.shape)
    per_key = (lambda x: np.full(dk, x[0])) if iso else (lambda x: x)
    for n in range(B):
        for h in range(H):
            ts = range(n * T, (n + 1) * T)
            lam_t, gate_t, dqh, dkh, G_t = {}, {}, {}, {}, {}
            # forward sweep: the precision chain and eta, dq^ = eta do
            lam = np.array(lam0[n, h], dtype=np.float64).reshape(nl)
            eta = eta0[n, h].copy()
            for t in ts:
                at, qt = np.reshape(a[t, h], nl), np.reshape(qn[t, h], nl)
                den = at * at + qt * lam
                gate_t[t] = at / den
                lam = lam / den + (beta[t, h] * np.sum(k[t, h] ** 2) / dk if iso else beta[t, h] * k[t, h] ** 2)
                lam_t[t] = lam
                eta = per_key(gate_t[t])[:, None] * eta + beta[t, h] * np.outer(k[t, h], v[t, h])
                dqh[t] = eta @ dout[t, h]
            # reverse sweep of the adjoint: dk^, dv, the gate term, dL/deta0
            d = dfe[n, h].copy()
            G = np.sum(dfe[n, h] * eta, axis=1)
            for t in reversed(ts):
                if t + 1 in gate_t:
                    d = per_key(gate_t[t + 1])[:, None] * d
                qhat = q[t, h] / per_key(lam_t[t])
                d = d + np.outer(qhat, dout[t, h])
                dkh[t] = d @ v[t, h]
                res["dv"][t, h] = d.T @ (beta[t, h] * k[t, h])
                G = G + qhat * dqh[t] - beta[t, h] * k[t, h] * dkh[t]
                G_t[t] = G
            res["deta0"][n, h] = per_key(gate_t[ts[0]])[:, None] * d
            # the precision chain in reverse
            dl = np.array(dfl[n, h], dtype=np.float64).reshape(nl)
            for t in reversed(ts):
                lp = lam_t[t - 1] if t - 1 in lam_t else np.array(lam0[n, h], dtype=np.float64).reshape(nl)
                at, qt = np.reshape(a[t, h], nl), np.reshape(qn[t, h], nl)
                sq = dqh[t] * q[t, h]
                Gt = G_t[t]
                if iso:
                    sq, Gt = np.array([sq.sum()]), np.array([Gt.sum()])
                dlt = dl - sq / lam_t[t] ** 2
                den = at * at + qt * lp
                dg = Gt * den / at
                dden = -(dlt * lp + dg * at) / den ** 2
                res["da"][t, h] = np.reshape(dg / den + 2 * at * dden, np.shape(a[t, h]))
                res["dqn"][t, h] = np.reshape(lp * dden, np.shape(qn[t, h]))
                dl = dlt / den + qt * dden
                # assembly
                dlk = per_key(dlt / dk if iso else dlt)
                res["dq"][t, h] = dqh[t] / per_key(lam_t[t])
                res["dk"][t, h] = beta[t, h] * dkh[t] + 2 * beta[t, h] * k[t, h] * dlk
                res["dbeta"][t, h] = np.sum(k[t, h] * (dkh[t] + k[t, h] * dlk))
            res["dlambda0"][n, h] = np.reshape(dl, np.shape(lam0[n, h]))
    return res


@pytest.mark.parametrize("iso", [False, True])
@pytest.mark.parametrize("strong", [False, True])
def test_sweeps_equal_the_oracles_reverse_mode(iso, strong):
    rng = np.random.default_rng(5 + iso + 2 * strong)
    B, T, H, dk, dv = 2, 24, 2, 8, 4
    Ntok, nl = B * T, () if iso else (dk,)
    f = lambda x: np.asarray(x, dtype=np.float32).astype(np.float64)  # noqa: E731
    x = dict(q=f(rng.standard_normal((Ntok, H, dk))), k=f(rng.standard_normal((Ntok, H, dk)) * 0.5),
             v=f(rng.standard_normal((Ntok, H, dv))),
             a=f(rng.uniform(0.02, 0.1, (Ntok, H) + nl) if strong else rng.uniform(0.3, 0.99, (Ntok, H) + nl)),
             qn=f(rng.uniform(0.0, 0.5, (Ntok, H) + nl)), beta=f(rng.uniform(0.2, 3.0, (Ntok, H))),
             dout=f(rng.standard_normal((Ntok, H, dv))), lam0=f(rng.uniform(0.5, 2.0, (B, H) + nl)),
             eta0=f(rng.standard_normal((B, H, dk, dv))), dfl=f(rng.standard_normal((B, H) + nl)),
             dfe=f(rng.standard_normal((B, H, dk, dv))))
    got = sweeps(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], x["dout"], x["lam0"], x["eta0"], x["dfl"],
                 x["dfe"], iso)
    want = oracle.backward(x["q"], x["k"], x["v"], x["a"], x["qn"], x["beta"], x["dout"], x["lam0"], x["eta0"],
                           x["dfl"], x["dfe"], B=B, T=T, iso=iso)
    for name, w in want.items():
        err = np.max(np.abs(got[name] - w) / (1.0 + np.abs(w)))
        assert err < 1e-9, (name, err)
