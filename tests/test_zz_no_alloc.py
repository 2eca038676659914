"""kla_forward_noalloc against kla_forward.

The no-allocation entry point serves callers that cannot call cudaMalloc
where they run the layer (allocator or pool callbacks, plug-ins whose host
owns every device allocation, fixed-footprint processes). It runs the same
forward pass with the library's fixed per-GPU scratch array as workspace.
This file is collected last so that a failure here leaves every other test
already run; it passes on its own in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2   # the bf16 parity tolerance of the other GPU tests


def _close(got, want):
    g = got.float().cpu().numpy().astype(np.float64)
    r = want.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - r) <= TOL * (1.0 + np.abs(r)))


def test_noalloc_matches_forward_on_two_calls(monkeypatch):
    # rows split into segments: the configuration whose forward pass needs scratch
    monkeypatch.setenv("KLA_SEGMENTS", "4")
    w = WORKLOADS[1].with_(B=2, H=4, T=1500)
    inp = make_inputs(w)
    d = {k: (t.cuda() if t is not None else None) for k, t in inp.items()}
    L = kla.lib()
    desc = kla.make_desc(w.B, w.T, w.H, w.dk, w.dv)
    need = L.kla_workspace_bytes(ctypes.byref(desc))
    assert 0 < need <= (32 << 20)
    ref = kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=w.B, T=w.T, final_state=True)
    torch.cuda.synchronize()
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full_like(ref[0], float("nan"))
        fl = torch.full_like(ref[1], float("nan"))
        fe = torch.full_like(ref[2], float("nan"))
        s = L.kla_forward_noalloc(ctypes.byref(desc), P(d["q"]), P(d["k"]), P(d["v"]), P(d["a"]), P(d["qn"]),
                                  P(d["beta"]), None, None, P(out), P(fl), P(fe), stream)
        assert s == kla.KLA_OK, kla.status_string(s)
        torch.cuda.synchronize()
        kla.check()
        _close(out, ref[0])
        _close(fl, ref[1])
        _close(fe, ref[2])


def test_noalloc_rejects_workspace_beyond_the_scratch_area():
    L = kla.lib()
    # 16 heads x 128k tokens at dk = dv = 128 need more workspace than the array holds
    desc = kla.make_desc(1, 131072, 16, 128, 128)
    assert L.kla_workspace_bytes(ctypes.byref(desc)) > (32 << 20)
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    s = L.kla_forward_noalloc(ctypes.byref(desc), p, p, p, p, p, p, None, None, p, None, None,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert s == kla.KLA_ERR_UNSUPPORTED
