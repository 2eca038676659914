"""kla_forward_noalloc against kla_forward.

The no-allocation entry point serves callers that cannot call cudaMalloc
where they run the layer (allocator or pool callbacks, plug-ins whose host
owns every device allocation, fixed-footprint processes). It runs the same
forward pass with the library's fixed per-GPU scratch array as workspace.

Because the scratch array keeps whatever the previous call left in it, the
test first runs a different problem (other inputs, other shape, another
segment count) through it, so that every scratch value the checked call reads
must have been written by that call itself. The checked call uses the same
plan and kernels as kla_forward, which use no atomics, so the two must agree
bit for bit.

This file is collected last so that a failure here leaves every other test
already run; it passes on its own in a fresh process as well.
"""
import ctypes

import pytest
import torch

from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs, random_state

pytestmark = pytest.mark.gpu


def _dev(inp):
    return {k: (t.cuda() if t is not None else None) for k, t in inp.items()}


def _noalloc(L, w, d, lam0, eta0):
    desc = kla.make_desc(w.B, w.T, w.H, w.dk, w.dv)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    N = w.B
    out = torch.full((w.tokens, w.H, w.dv), float("nan"), dtype=torch.bfloat16, device="cuda")
    fl = torch.full((N, w.H, w.dk), float("nan"), device="cuda")
    fe = torch.full((N, w.H, w.dk, w.dv), float("nan"), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    s = L.kla_forward_noalloc(ctypes.byref(desc), P(d["q"]), P(d["k"]), P(d["v"]), P(d["a"]), P(d["qn"]),
                              P(d["beta"]), P(lam0), P(eta0), P(out), P(fl), P(fe), stream)
    assert s == kla.KLA_OK, kla.status_string(s)
    torch.cuda.synchronize()
    kla.check()
    return out, fl, fe


def test_noalloc_matches_forward_after_other_work_in_the_scratch(monkeypatch):
    L = kla.lib()
    # the checked problem: rows split into segments, the configuration whose
    # forward pass needs scratch
    w = WORKLOADS[1].with_(B=2, H=4, T=1500)
    d = _dev(make_inputs(w))
    lam0, eta0 = (t.cuda() for t in random_state(w, w.B, seed=31))
    desc = kla.make_desc(w.B, w.T, w.H, w.dk, w.dv)
    monkeypatch.setenv("KLA_SEGMENTS", "4")
    need = L.kla_workspace_bytes(ctypes.byref(desc))
    assert 0 < need <= kla.NOALLOC_SCRATCH_BYTES
    ref = kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], lam0, eta0, B=w.B, T=w.T,
                      final_state=True)
    torch.cuda.synchronize()
    kla.check()
    # other work through the scratch array: different inputs, shape and segment count
    w2 = WORKLOADS[1].with_(B=3, H=5, T=2300, seed=77)
    d2 = _dev(make_inputs(w2))
    lam2, eta2 = (t.cuda() for t in random_state(w2, w2.B, seed=78))
    for segs in ("7", "3"):
        monkeypatch.setenv("KLA_SEGMENTS", segs)
        _noalloc(L, w2, d2, lam2, eta2)
        # two calls of the checked problem in a row after it
        monkeypatch.setenv("KLA_SEGMENTS", "4")
        for _ in range(2):
            out, fl, fe = _noalloc(L, w, d, lam0, eta0)
            assert torch.equal(out, ref[0])
            assert torch.equal(fl, ref[1])
            assert torch.equal(fe, ref[2])


def test_noalloc_rejects_workspace_beyond_the_scratch_area():
    L = kla.lib()
    # 16 heads x 128k tokens at dk = dv = 128 need more workspace than the array holds
    desc = kla.make_desc(1, 131072, 16, 128, 128)
    assert L.kla_workspace_bytes(ctypes.byref(desc)) > kla.NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    s = L.kla_forward_noalloc(ctypes.byref(desc), p, p, p, p, p, p, None, None, p, None, None,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert s == kla.KLA_ERR_UNSUPPORTED
