"""Pins of the prologue oracle (1-D causal conv + SiLU, L2 norm, gates)."""
import numpy as np
import pytest

import oracle


def _inputs(rng, Ntok, H, dk, dv, W=4):
    x = lambda *s: rng.standard_normal(s)  # noqa: E731
    return dict(xq=x(Ntok, H, dk), xk=x(Ntok, H, dk), xv=x(Ntok, H, dv), xa=x(Ntok, H, dk), xqn=x(Ntok, H, dk),
                xbeta=x(Ntok, H), wq=x(H, dk, W), wk=x(H, dk, W), wv=x(H, dv, W), bq=x(H, dk), bk=x(H, dk),
                bv=x(H, dv))


def test_identity_conv_reduces_to_the_activations():
    # a kernel (0, ..., 0, 1) and no bias is the identity: q = l2norm(silu(xq)), v = silu(xv)
    rng = np.random.default_rng(0)
    p = _inputs(rng, 20, 2, 8, 5)
    for w in ("wq", "wk", "wv"):
        p[w][:] = 0.0
        p[w][..., -1] = 1.0
    p["bq"] = p["bk"] = p["bv"] = None
    r = oracle.prologue(**p, B=1, T=20)
    s = p["xq"] / (1 + np.exp(-p["xq"]))
    np.testing.assert_allclose(r["q"], s / np.sqrt((s * s).sum(-1, keepdims=True) + oracle.PROLOGUE_EPS), rtol=1e-13)
    np.testing.assert_allclose(r["v"], p["xv"] / (1 + np.exp(-p["xv"])), rtol=1e-13)


def test_conv_is_numpys_causal_convolution_per_channel():
    rng = np.random.default_rng(1)
    T, H, dk, dv = 30, 2, 4, 3
    p = _inputs(rng, T, H, dk, dv)
    p["bq"] = None
    r = oracle.prologue(**p, B=1, T=T)
    for h in range(H):
        for c in range(dk):
            # np.convolve flips the kernel: y[t] = sum_w w[W-1-w'] x[t-w'] = our taps in reverse
            y = np.convolve(p["xq"][:, h, c], p["wq"][h, c, ::-1])[:T]
            s = y / (1 + np.exp(-y))
            want = s  # before the norm: compare after undoing it with the same row norm
            got = r["q"][:, h, c]
            norm = np.sqrt(sum((lambda z: z / (1 + np.exp(-z)))(np.convolve(p["xq"][:, h, cc], p["wq"][h, cc, ::-1])[:T]) ** 2
                               for cc in range(dk)) + oracle.PROLOGUE_EPS)
            np.testing.assert_allclose(got, want / norm, rtol=1e-12, atol=1e-14)


def test_gates_closed_forms_and_unit_norms():
    rng = np.random.default_rng(2)
    p = _inputs(rng, 16, 3, 8, 8)
    p["xa"][0, 0, 0] = 0.0
    p["xqn"][0, 0, 0] = 0.0
    p["xbeta"][0, 0] = 0.0
    p["xqn"][1, 0, 0] = 50.0
    p["xqn"][2, 0, 0] = -50.0
    r = oracle.prologue(**p, B=2, T=8)
    assert r["a"][0, 0, 0] == 0.5 and r["beta"][0, 0] == 0.5
    np.testing.assert_allclose(r["qn"][0, 0, 0], np.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(r["qn"][1, 0, 0], 50.0, rtol=1e-15)          # softplus(y) ~ y for large y
    np.testing.assert_allclose(r["qn"][2, 0, 0], np.exp(-50.0), rtol=1e-12)  # ~ e^y for very negative y
    assert np.all((r["a"] > 0) & (r["a"] < 1)) and np.all(r["qn"] > 0)
    nq = np.sqrt((r["q"] ** 2).sum(-1))
    assert np.all(nq <= 1.0 + 1e-12) and np.all(nq > 0.99)


def test_packed_sequences_restart_the_convolution():
    rng = np.random.default_rng(3)
    p = _inputs(rng, 25, 2, 4, 4)
    cu = np.array([0, 7, 8, 25])
    r = oracle.prologue(**p, cu_seqlens=cu)
    for s, e in zip(cu[:-1], cu[1:]):
        part = {k: (v[s:e] if v is not None and v.ndim >= 2 and v.shape[0] == 25 else v) for k, v in p.items()}
        alone = oracle.prologue(**part, B=1, T=int(e - s))
        for key in ("q", "k", "v", "a", "qn", "beta"):
            np.testing.assert_allclose(r[key][s:e], alone[key], rtol=1e-13, atol=1e-15)
