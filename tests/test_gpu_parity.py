"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.

Bar (per element, out / final_lambda / final_eta / lambda trajectory):
    |gpu - oracle| <= tol * (1 + |oracle|)
with tol = 2e-2 for bf16 inputs (fp32 accumulation, bf16 tensor-core operands)
and tol = 1e-4 for fp32 inputs.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from bayesian_filter_scan_b200 import kla
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs, random_state

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "fp32": 1e-4}


# max scaled error of every comparison, printed in the session summary
ERRORS = []


def close(got, want, tol, what=""):
    got = got.detach().float().cpu().numpy().astype(np.float64) if hasattr(got, "detach") else got
    err = np.abs(got - want) / (1.0 + np.abs(want))
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]
    ERRORS.append((test, what, float(np.nanmax(err)) if err.size else 0.0, tol))
    bad = ~(err <= tol)
    assert not bad.any(), "%s: %d/%d elements off, max scaled err %.3g at %s" % (
        what, int(bad.sum()), bad.size, float(np.nanmax(err)), np.unravel_index(np.nanargmax(err), err.shape))


def to_dev(inp):
    return {k: (v.cuda() if v is not None else None) for k, v in inp.items()}


def run(w, inp, lam0=None, eta0=None, final=True):
    d = to_dev(inp)
    lam0 = lam0.cuda() if lam0 is not None else None
    eta0 = eta0.cuda() if eta0 is not None else None
    r = kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], lam0, eta0,
                    cu_seqlens=d["cu_seqlens"], B=w.B, T=w.T, mode=w.mode, final_state=final)
    torch.cuda.synchronize()
    kla.check()
    return r


def compare(w, inp, lam0=None, eta0=None, units=None):
    res = run(w, inp, lam0, eta0)
    x = dict(inp)
    x["lambda0"], x["eta0"] = lam0, eta0
    ref = oracle.forward_inputs(x, w, units=units)
    tol = TOL[w.dtype]
    out, fl, fe = res
    if units is None:
        close(out, ref["out"], tol, "out")
        close(fl, ref["final_lambda"], tol, "final_lambda")
        close(fe, ref["final_eta"], tol, "final_eta")
    else:
        H = w.H
        for u in range(*units):
            n, h = divmod(u, H)
            s, e = n * w.T, (n + 1) * w.T
            close(out[s:e, h], ref["out"][s:e, h], tol, "out unit %d" % u)
            close(fl[n, h], ref["final_lambda"][n, h], tol, "final_lambda unit %d" % u)
            close(fe[n, h], ref["final_eta"][n, h], tol, "final_eta unit %d" % u)
    return res


def test_tiny_fp32_workload():
    w = WORKLOADS[0]
    compare(w, make_inputs(w))


def test_small_layer_workload_full():
    w = WORKLOADS[1]
    compare(w, make_inputs(w))


@pytest.mark.parametrize("segments", ["1", "3", "8"])
def test_segmented_path_matches(monkeypatch, segments):
    monkeypatch.setenv("KLA_SEGMENTS", segments)
    w = WORKLOADS[1].with_(B=2, H=3, T=2000)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=21)
    compare(w, inp, lam0, eta0)


@pytest.mark.parametrize("segments", ["2", "24"])
def test_long_and_many_segments(monkeypatch, segments):
    # two long segments (24 blocks each: the correction pass runs its zero test
    # over several chunks per CTA) and 24 short ones (two blocks each: 23
    # segment-start beliefs chained before the last segment)
    monkeypatch.setenv("KLA_SEGMENTS", segments)
    w = WORKLOADS[1].with_(B=1, H=2, T=3000)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=23)
    compare(w, inp, lam0, eta0)


def test_correction_zero_test(monkeypatch):
    # 64 rows x heads in two segments of 32 blocks: correction CTAs of four
    # chunks, so the zero test over the chunks runs
    monkeypatch.setenv("KLA_SEGMENTS", "2")
    w = WORKLOADS[1].with_(B=4, H=16, T=4096)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=29)
    compare(w, inp, lam0, eta0)


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 127, 257, 1000])
def test_ragged_lengths(T):
    w = WORKLOADS[1].with_(B=2, H=2, T=T)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=T)
    compare(w, inp, lam0, eta0)


@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 256), (32, 64), (64, 128), (128, 64), (128, 128),
                                   (128, 256)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_head_dims(dk, dv, dtype):
    w = WORKLOADS[2].with_(B=1, H=2, T=200, dk=dk, dv=dv, dtype=dtype)
    compare(w, make_inputs(w))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_isotropic_varlen_small(dtype):
    w = WORKLOADS[4].with_(B=2, H=3, T=1500, len_lo=1, len_hi=400, dtype=dtype)
    inp = make_inputs(w)
    N = inp["cu_seqlens"].numel() - 1
    lam0, eta0 = random_state(w, N, seed=3)
    compare(w, inp, lam0, eta0)


def test_diagonal_varlen_small():
    w = WORKLOADS[1].with_(B=2, H=2, T=700, varlen=True, len_lo=1, len_hi=300)
    compare(w, make_inputs(w))


@pytest.mark.parametrize("len_hi", [9, 30])
def test_many_packed_sequences(len_hi):
    # ~1700 sequences (beyond the 1024 the device ranks by length: launched in
    # input order) and ~600 (ranked, longest first); lengths 1..len_hi
    w = WORKLOADS[1].with_(B=1, H=2, T=9000, varlen=True, len_lo=1, len_hi=len_hi)
    inp = make_inputs(w)
    N = inp["cu_seqlens"].numel() - 1
    assert (N > 1024) == (len_hi == 9)
    lam0, eta0 = random_state(w, N, seed=5)
    compare(w, inp, lam0, eta0)


def test_isotropic_unpacked_segmented(monkeypatch):
    monkeypatch.setenv("KLA_SEGMENTS", "4")
    w = WORKLOADS[4].with_(B=1, H=2, T=3000, varlen=False)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, 1, seed=8)
    compare(w, inp, lam0, eta0)


def test_precision_trajectory():
    for w in (WORKLOADS[1].with_(B=2, H=2, T=1000), WORKLOADS[4].with_(B=1, H=2, T=3000, len_lo=100, len_hi=900)):
        inp = make_inputs(w)
        d = to_dev(inp)
        lam = kla.precision(d["k"], d["a"], d["qn"], d["beta"], cu_seqlens=d["cu_seqlens"], B=w.B, T=w.T,
                            mode=w.mode)
        torch.cuda.synchronize()
        ref = oracle.forward_inputs(inp, w, want_lambda=True, want_out=False, want_final=False)
        close(lam, ref["lambda"], 1e-4, "lambda")


def test_decode_steps_equal_forward():
    w = WORKLOADS[1].with_(B=3, H=2, T=20)
    inp = make_inputs(w)
    lam0, eta0 = random_state(w, w.B, seed=2)
    full = oracle.forward(inp["q"], inp["k"], inp["v"], inp["a"], inp["qn"], inp["beta"], lam0, eta0, B=w.B, T=w.T)
    d = to_dev(inp)
    lam, eta = lam0.clone().cuda(), eta0.clone().cuda()
    H = w.H
    rows = lambda x: x.view(w.B, w.T, *x.shape[1:])
    outs = []
    for t in range(w.T):
        sl = lambda x: rows(x)[:, t].contiguous()
        outs.append(kla.decode_step(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["a"]), sl(d["qn"]),
                                    sl(d["beta"]), lam, eta))
    torch.cuda.synchronize()
    got = torch.stack(outs, 1).reshape(w.B * w.T, H, w.dv)
    close(got, full["out"], 2e-2, "decode out")
    close(lam, full["final_lambda"], 1e-4, "decode lambda")
    close(eta, full["final_eta"], 2e-2, "decode eta")


def test_split_call_hand_off_on_gpu():
    w = WORKLOADS[1].with_(B=1, H=2, T=1500)
    inp = make_inputs(w)
    d = to_dev(inp)
    T1 = 577
    half = lambda x, s, e: x[s:e].contiguous()
    o1, l1, e1 = kla.forward(*(half(d[n], 0, T1) for n in ("q", "k", "v", "a", "qn", "beta")), B=1, T=T1,
                             final_state=True)
    o2, l2, e2 = kla.forward(*(half(d[n], T1, w.T) for n in ("q", "k", "v", "a", "qn", "beta")), l1, e1,
                             B=1, T=w.T - T1, final_state=True)
    ref = oracle.forward_inputs(inp, w)
    close(torch.cat([o1, o2]), ref["out"], 2e-2, "split out")
    close(l2, ref["final_lambda"], 2e-2, "split lambda")
    close(e2, ref["final_eta"], 2e-2, "split eta")


def test_host_buffer_entry_point_matches_device_entry_point():
    w = WORKLOADS[1].with_(B=2, H=2, T=600)
    inp = make_inputs(w)
    dev_out, dev_fl, dev_fe = run(w, inp)
    pin = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    desc = kla.make_desc(w.B, w.T, w.H, w.dk, w.dv)
    out = torch.empty(w.B * w.T, w.H, w.dv, dtype=torch.bfloat16).pin_memory()
    fl = torch.empty(w.B, w.H, w.dk).pin_memory()
    fe = torch.empty(w.B, w.H, w.dk, w.dv).pin_memory()
    kla.forward_host(desc, pin["q"], pin["k"], pin["v"], pin["a"], pin["qn"], pin["beta"], out,
                     final_lambda=fl, final_eta=fe)
    assert torch.equal(out, dev_out.cpu())
    assert torch.equal(fl, dev_fl.cpu()) and torch.equal(fe, dev_fe.cpu())


def test_deterministic():
    w = WORKLOADS[1].with_(B=2, H=4, T=1500)
    inp = make_inputs(w)
    a = run(w, inp)
    b = run(w, inp)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_empty_input_is_noop():
    w = WORKLOADS[1].with_(B=1, H=2, T=0)
    inp = make_inputs(w)
    d = to_dev(inp)
    out = kla.forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], B=1, T=0)
    assert out.numel() == 0


# ---- full-size workloads, in the launch configuration the benchmark times ---

def test_layer_workload_full_size():
    w = WORKLOADS[2]
    compare(w, make_inputs(w))


def test_long_context_workload_sampled_heads():
    w = WORKLOADS[3]
    compare(w, make_inputs(w), units=(0, 2))


def test_isotropic_varlen_stress_workload_full():
    w = WORKLOADS[4]
    compare(w, make_inputs(w))
