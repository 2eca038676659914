"""Host-side helpers of bench.py: the algorithmic byte counts its roofline
lines divide by, and the bounded token prefix its prologue CPU baseline times."""
import numpy as np
import pytest
import torch

import bench
import oracle
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs


def test_algorithmic_bytes_per_token_head():
    w = WORKLOADS[2]                      # d = 128, bf16, diagonal
    # forward: q, k, v bf16 (3 x 256), a, qn fp32 (2 x 512), beta, out bf16 (256)
    assert bench.bytes_per_token_head(w) == 3 * 256 + 2 * 512 + 4 + 256 == 2052
    # Moebius reduce: k bf16, a, qn fp32, beta
    assert bench.scan_bytes_per_token_head(w) == 256 + 2 * 512 + 4 == 1284
    # prologue: the six pre-activations read and the six outputs written
    assert bench.prologue_bytes_per_token_head(w) == 2 * (3 * 256 + 2 * 512 + 4) == 3592
    # backward: the inputs and dout read, every gradient written in fp32
    assert bench.backward_bytes_per_token_head(w) == 2052 + 4 * (2 * 128 + 128 + 2 * 128 + 1) == 4616
    iso = WORKLOADS[4]                    # dk = 64, dv = 128, isotropic gates
    assert bench.bytes_per_token_head(iso) == 2 * (2 * 64 + 2 * 128) + 2 * 4 + 4


@pytest.mark.parametrize("wid", [1, 4])
def test_prologue_sample_is_the_prefix_problem(wid):
    w = WORKLOADS[wid].with_(B=2, H=2, T=300) if wid == 1 else \
        WORKLOADS[4].with_(B=1, H=2, T=900, len_lo=1, len_hi=200, dk=16, dv=16)
    inp = make_inputs(w)
    g = torch.Generator().manual_seed(1)
    Ntok, H, dk, dv = inp["q"].shape[0], w.H, w.dk, w.dv
    gate = (Ntok, H) if w.mode == "iso" else (Ntok, H, dk)
    r = lambda *s: torch.randn(*s, generator=g)  # noqa: E731
    x = {"xq": r(Ntok, H, dk), "xk": r(Ntok, H, dk), "xv": r(Ntok, H, dv), "xa": r(*gate), "xqn": r(*gate),
         "xbeta": r(Ntok, H), "wq": r(H, dk, 4), "wk": r(H, dk, 4), "wv": r(H, dv, 4),
         "bq": r(H, dk), "bk": r(H, dk), "bv": r(H, dv)}
    cu = inp["cu_seqlens"]
    full = oracle.prologue(**x, cu_seqlens=cu, B=None if cu is not None else w.B, T=None if cu is not None else w.T)
    for n in (1, 150, 300, 451, Ntok):
        xs, bounds = bench._prologue_sample(x, cu, w, n)
        assert bounds[0] == 0 and bounds[-1] == n and np.all(np.diff(bounds) > 0)
        part = oracle.prologue(**xs, cu_seqlens=bounds)
        for name in ("q", "k", "v", "a", "qn", "beta"):
            np.testing.assert_allclose(part[name], full[name][:n], rtol=0, atol=1e-12)
