#!/usr/bin/env python
"""Throughput benchmark of the Kalman linear-attention forward pass on B200.

One step = one kla_forward call over one batch of the workload (the whole hot
path: Moebius precision scan, state passing, chunked tensor-core pass) with
inputs resident in HBM. The default workload is the largest single-GPU one,
the 128k-token long context (B=1, H=16, T=131072, dk=dv=128, final state
returned). Prints ONE JSON line (rank 0):

  value        tokens/s (B*T per second, all ranks together), device-timed with
               CUDA events on the launching stream around each call, L2 flushed
               (512 MiB write) between timed steps, max over ranks;
  e2e          the same metric through kla_forward_host: pinned host inputs
               copied in, forward, output copied back, inside the timed region;
  roofline     the dominant kernel (the chunk kernel walking whole rows, or the
               segments of split rows) against the measured HBM copy bandwidth:
               algorithmic bytes (inputs read once, output written once) / its
               event-timed duration;
  roofline_scan the Moebius precision scan's block reduction (rows split into
               segments) against the same peak;
  max_err      the largest scaled error |gpu - oracle| / (1 + |oracle|) of the
               timed output on the units the CPU baseline computed;
  cpu_baseline the CPU oracle (plain fp64 C, OpenMP) on a bounded sample of
               the same workload, on this host's cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 3] [--impl reference]
  python bench.py --variant kdn [--workload 2]   (the Kalman Delta Network residual write:
               a separate line with the same timing rules, kla_kdn_forward)

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
the workload (independent sequences; no collective on the data path), so the
scaling is weak; value = ranks * tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "KLA forward tokens/s per layer (B*T/s) on 1 B200; % of HBM / bf16 TC roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = 3
FLUSH_BYTES = 512 << 20
SWEEP_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
TOL = {"bf16": 2e-2, "fp32": 1e-4}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def workload_label(w):
    s = "%s B=%d H=%d T=%d dk=%d dv=%d %s %s" % (w.name, w.B, w.H, w.T, w.dk, w.dv, w.dtype, w.mode)
    return s + (" varlen" if w.varlen else "")


def bytes_per_token_head(w) -> int:
    """Algorithmic bytes of the forward pass per (token, head): every input
    read once and the output written once."""
    es = 2 if w.dtype == "bf16" else 4
    nl = 1 if w.mode == "iso" else w.dk
    return es * (2 * w.dk + 2 * w.dv) + 4 * 2 * nl + 4


def scan_bytes_per_token_head(w) -> int:
    """Algorithmic bytes of the Moebius block reduction per (token, head): the
    key, the decay and process noise, and the value precision, read once."""
    es = 2 if w.dtype == "bf16" else 4
    nl = 1 if w.mode == "iso" else w.dk
    return es * w.dk + 4 * 2 * nl + 4


def flops_per_token_head(w) -> int:
    """The recurrence's own arithmetic: rank-1 state update and readout."""
    return 4 * w.dk * w.dv


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def source_hash(name: str) -> str:
    with open(os.path.join(ROOT, "bayesian_filter_scan_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_record(wid, kernel_file="kla_chunk_tc.cu"):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "chunk_kernel_traffic.json")
    try:
        rec = json.load(open(path)).get(str(wid))
    except Exception:
        return None
    if not rec or rec.get("kernel_sha") != source_hash(kernel_file):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, read through
    NVML every 5 ms on a background thread while the timed region runs (read
    only: no clock or other setting is changed)."""

    NAMES = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
             ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
             ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
             ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.err = None
        self._stop = threading.Event()
        self._thr = None
        self.nv = None
        self.handle = None
        self.max_mhz = None

    def _open(self):
        import pynvml as nv
        nv.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        h = None
        try:
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            h = nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            h = nv.nvmlDeviceGetHandleByIndex(self.dev)
        self.nv, self.handle = nv, h
        self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

    def _run(self):
        nv, h = self.nv, self.handle
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((mhz, rs))
            except Exception as e:  # noqa: BLE001
                self.err = str(e)
                return
            time.sleep(0.005)

    def start(self):
        try:
            self._open()
        except Exception as e:  # noqa: BLE001
            self.err = "NVML unavailable: %s" % e
            return
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()

    def stop(self):
        if self._thr is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no sampler"], "samples": 0}
        self._stop.set()
        self._thr.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [self.err or "no samples"],
                    "samples": 0}
        reasons = sorted({name for _, rs in self.samples for name, attr in self.NAMES
                          if rs & int(getattr(self.nv, attr, 0))})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(m for m, _ in self.samples), "reasons": reasons,
                "samples": len(self.samples), "source": "NVML, every 5 ms during the timed region"}


def rank_seed(w, rank: int) -> int:
    """Each rank draws its own batch (independent sequences): weak scaling."""
    return w.seed + 7919 * rank


def aggregate(world: int, tokens_per_rank: int, local_ms_total: float, steps: int, dist=None, device="cuda"):
    """Max-over-ranks timing and the whole-job throughput (tokens/s)."""
    t = torch.tensor([local_ms_total], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_per_step = t.item() / steps
    return ms_per_step, world * tokens_per_rank / (ms_per_step * 1e-3)


def _units_total(w, inp):
    return (inp["cu_seqlens"].numel() - 1 if inp["cu_seqlens"] is not None else w.B) * w.H


def _unit_tokens(w, inp, n_units):
    """Tokens (summed over heads, / H) of the first n_units (sequence, head) units."""
    if inp["cu_seqlens"] is None:
        return n_units * w.T / w.H
    cu = inp["cu_seqlens"].tolist()
    return sum(cu[u // w.H + 1] - cu[u // w.H] for u in range(n_units)) / w.H


def sample_units(w, inp, target_s):
    """How many (sequence, head) units of the workload the oracle computes in
    about target_s seconds on this host's cores (at least one)."""
    import oracle
    t1 = time.perf_counter()
    oracle.forward_inputs(inp, w, units=(0, 1), want_final=False)
    per_unit = max(time.perf_counter() - t1, 1e-4)
    return int(max(1, min(_units_total(w, inp), target_s / per_unit * oracle.max_threads())))


def cpu_baseline(w, inp, target_s=12.0):
    """The oracle, as it stands, on a bounded sample of (row, head) units.
    Returns the baseline record and the oracle's result on those units."""
    import oracle
    n_units = sample_units(w, inp, target_s)
    reps, t, ref = 0, 0.0, None
    while reps == 0 or t < 2.0:       # repeat a small sample for a stable time
        t0 = time.perf_counter()
        ref = oracle.forward_inputs(inp, w, units=(0, n_units), want_final=True)
        t += time.perf_counter() - t0
        reps += 1
    t /= reps
    rec = {"value": _unit_tokens(w, inp, n_units) / t, "unit": UNIT, "cores": oracle.max_threads(),
           "kind": "oracle",
           "sample": "%d of %d (row, head) units of the workload, fp64 C oracle, %.3f s per pass, %d passes" % (
               n_units, _units_total(w, inp), t, reps)}
    return rec, ref, n_units


def scaled_err(got: torch.Tensor, want: np.ndarray) -> float:
    """max |got - want| / (1 + |want|), computed in slices to bound host memory."""
    g = got.reshape(got.shape[0], -1)
    r = want.reshape(want.shape[0], -1)
    worst = 0.0
    step = max(1, (1 << 24) // max(1, g.shape[1]))
    for s in range(0, g.shape[0], step):
        gs = g[s:s + step].float().cpu().numpy().astype(np.float64)
        rs = r[s:s + step]
        worst = max(worst, float(np.max(np.abs(gs - rs) / (1.0 + np.abs(rs)))) if gs.size else 0.0)
    return worst


def max_err(w, inp, ref, n_units, out, fl, fe):
    """Scaled error of the GPU results against the oracle on its sampled units."""
    H = w.H
    cu = inp["cu_seqlens"].tolist() if inp["cu_seqlens"] is not None else None
    e_out = e_fl = e_fe = 0.0
    for u in range(n_units):
        n, h = divmod(u, H)
        s, e = (cu[n], cu[n + 1]) if cu else (n * w.T, (n + 1) * w.T)
        e_out = max(e_out, scaled_err(out[s:e, h], ref["out"][s:e, h]))
        if fl is not None:
            e_fl = max(e_fl, scaled_err(fl[n:n + 1, h], ref["final_lambda"][n:n + 1, h]))
            e_fe = max(e_fe, scaled_err(fe[n:n + 1, h], ref["final_eta"][n:n + 1, h]))
    res = {"out": e_out, "units": n_units, "tol": TOL[w.dtype],
           "definition": "max |gpu - oracle| / (1 + |oracle|) over the sampled units"}
    if fl is not None:
        res["final_lambda"], res["final_eta"] = e_fl, e_fe
    return res


def arm_config(w, world):
    """The workload's `config` object, identical on both arms."""
    return {"workload": workload_label(w), "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv,
            "mode": w.mode, "varlen": w.varlen, "final_state": w.final_state,
            "tokens_per_step_per_gpu": w.tokens,
            "l2": "flushed between timed steps (512 MiB device write, then 256 MiB read)",
            "parallelism": "dp%d" % world}


KDN_METRIC = "KDN residual-write forward tokens/s per layer (B*T/s) on 1 B200; % of HBM"


def run_kdn(args, w):
    """The Kalman Delta Network residual write (kla_kdn_forward) on the
    workload: one launch per step, device-timed with L2 flushed between steps,
    against the same algorithmic bytes as the KLA forward (inputs once, output
    once); end to end with the inputs copied in from pinned host memory and the
    output copied back inside the timed region; the fp64 oracle on a bounded
    sample of units as the CPU baseline. One GPU (the path shards like the KLA
    forward: replicas)."""
    from bayesian_filter_scan_b200 import kla
    torch.cuda.set_device(0)
    kla.lib()
    inp = make_inputs(w, seed=rank_seed(w, 0))
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    H, dv = w.H, w.dv
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    sweep = torch.ones(SWEEP_BYTES // 4, dtype=torch.float32, device="cuda")
    out = torch.empty(w.tokens, H, dv, dtype=dev["q"].dtype, device="cuda")

    def run(d, o):
        return kla.kdn_forward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], cu_seqlens=d["cu_seqlens"],
                               B=w.B, T=w.T, mode=w.mode, out=o)

    def flush_l2():
        flush.fill_(1)
        sweep.sum()
    for _ in range(args.warmup):
        flush_l2()
        run(dev, out)
    torch.cuda.synchronize()
    kla.check()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(0)
    clocks.start()
    for e0, e1 in ev:
        flush_l2()
        e0.record(stream)
        run(dev, out)
        e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    kla.check()
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    value = w.tokens / (ms * 1e-3)
    # end to end: pinned inputs in, output out, inside the timed region
    pin = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    hout = torch.empty(w.tokens, H, dv, dtype=inp["q"].dtype).pin_memory()
    dbuf = {k: (torch.empty_like(v, device="cuda") if v is not None else None) for k, v in inp.items()}
    h_in = sum(t.numel() * t.element_size() for k_, t in pin.items()
               if t is not None and k_ in ("q", "k", "v", "a", "qn", "beta", "cu_seqlens"))
    e_t, e_steps = 0.0, max(3, min(args.e2e_steps, args.steps))
    for i in range(e_steps + 2):
        flush_l2()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for k_, t in pin.items():
            if t is not None:
                dbuf[k_].copy_(t, non_blocking=True)
        run(dbuf, out)
        hout.copy_(out, non_blocking=True)
        a1.record(stream)
        a1.synchronize()
        if i >= 2:
            e_t += a0.elapsed_time(a1)
    e2e_value = w.tokens / (e_t / e_steps * 1e-3)
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    alg_bytes = bytes_per_token_head(w) * w.tokens * H
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    cfg = arm_config(w, 1)
    cfg["variant"] = "kdn-residual-write"
    res = {
        "metric": KDN_METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": cfg,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "kdn_walk_kernel (CUDA cores, one CTA per row x head x 32 value columns)",
                     "alg_bytes_per_launch": alg_bytes, "launch_ms": ms,
                     "alg_bytes_per_token_head": bytes_per_token_head(w),
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_src},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h_in,
                "d2h_bytes_per_step": hout.numel() * hout.element_size()},
        "gpu_launches": args.steps, "clocks": clk,
    }
    if not args.no_cpu_baseline:
        import oracle
        t1 = time.perf_counter()
        oracle.kdn_forward_inputs(inp, w, units=(0, 1))
        per_unit = max(time.perf_counter() - t1, 1e-4)
        n_units = int(max(1, min(_units_total(w, inp), 12.0 / per_unit * oracle.max_threads())))
        t0 = time.perf_counter()
        ref = oracle.kdn_forward_inputs(inp, w, units=(0, n_units))
        t = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": _unit_tokens(w, inp, n_units) / t, "unit": UNIT,
                               "cores": oracle.max_threads(), "kind": "oracle",
                               "sample": "%d of %d (row, head) units, fp64 C oracle (residual write), %.3f s" % (
                                   n_units, _units_total(w, inp), t)}
        cu = inp["cu_seqlens"].tolist() if inp["cu_seqlens"] is not None else None
        worst = 0.0
        for u in range(n_units):
            n, h = divmod(u, H)
            s0, s1 = (cu[n], cu[n + 1]) if cu else (n * w.T, (n + 1) * w.T)
            worst = max(worst, scaled_err(out[s0:s1, h], ref["out"][s0:s1, h]))
        res["max_err"] = {"out": worst, "units": n_units, "tol": 2e-2 if w.dtype == "bf16" else 1e-4}
    print(json.dumps(res))


PRO_METRIC = "mixer prologue (conv + SiLU, L2 norm, gates) tokens/s per layer (B*T/s) on 1 B200; % of HBM"


def prologue_bytes_per_token_head(w) -> int:
    """Algorithmic bytes of the prologue per (token, head): every
    pre-activation read once, every output written once."""
    es = 2 if w.dtype == "bf16" else 4
    nl = 1 if w.mode == "iso" else w.dk
    return 2 * (es * (2 * w.dk + w.dv) + 4 * 2 * nl + 4)


def _prologue_sample(x, cu, w, n):
    """The first n tokens of the flattened token axis as a problem of their
    own (the rows or packed sequences that start inside it, the last one cut
    at n): arguments for oracle.prologue."""
    xs = {k: (v[:n] if k.startswith("x") else v) for k, v in x.items()}
    if cu is None:
        T = w.T
        bounds = list(range(0, n, T)) + [n]
    else:
        bounds = [c for c in cu.tolist() if c < n] + [n]
    return xs, np.asarray(bounds, dtype=np.int64)


def run_prologue(args, w):
    """kla_prologue on the workload's shape with synthetic pre-activations and
    conv weights (width 4): device-timed with L2 flushed between steps,
    against its algorithmic bytes and the measured HBM peak; end to end with
    the pre-activations copied in from pinned host memory and the six outputs
    copied back inside the timed region; the numpy fp64 oracle on a bounded
    prefix of the tokens as the CPU baseline."""
    from bayesian_filter_scan_b200 import kla
    torch.cuda.set_device(0)
    kla.lib()
    inp = make_inputs(w, seed=rank_seed(w, 0))
    g = torch.Generator().manual_seed(w.seed)
    dt = inp["q"].dtype
    Ntok, H, dk, dv = inp["q"].shape[0], w.H, w.dk, w.dv
    gate = (Ntok, H) if w.mode == "iso" else (Ntok, H, dk)
    r = lambda *s_: torch.randn(*s_, generator=g)  # noqa: E731
    x = {"xq": r(Ntok, H, dk).to(dt), "xk": r(Ntok, H, dk).to(dt), "xv": r(Ntok, H, dv).to(dt),
         "xa": r(*gate) + 2.0, "xqn": r(*gate) - 2.0, "xbeta": r(Ntok, H),
         "wq": r(H, dk, 4) / 2, "wk": r(H, dk, 4) / 2, "wv": r(H, dv, 4) / 2,
         "bq": r(H, dk) * 0.1, "bk": r(H, dk) * 0.1, "bv": r(H, dv) * 0.1}
    d = {k: v.cuda().contiguous() for k, v in x.items()}
    cu = inp["cu_seqlens"].cuda() if inp["cu_seqlens"] is not None else None
    outs = (torch.empty_like(d["xq"]), torch.empty_like(d["xk"]), torch.empty_like(d["xv"]),
            torch.empty_like(d["xa"]), torch.empty_like(d["xqn"]), torch.empty_like(d["xbeta"]))
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    sweep = torch.ones(SWEEP_BYTES // 4, dtype=torch.float32, device="cuda")

    def step():
        flush.fill_(1)
        sweep.sum()
        kla.prologue(**d, cu_seqlens=cu, B=None if cu is not None else w.B, T=None if cu is not None else w.T,
                     mode=w.mode, out=outs)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(0)
    clocks.start()
    ts = []
    for _ in range(args.steps):
        flush.fill_(1)
        sweep.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kla.prologue(**d, cu_seqlens=cu, B=None if cu is not None else w.B, T=None if cu is not None else w.T,
                     mode=w.mode, out=outs)
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = statistics.mean(a_.elapsed_time(b_) for a_, b_ in ts)
    kla.check()
    # end to end: pinned pre-activations in, the six outputs out, inside the timed region
    names = ("xq", "xk", "xv", "xa", "xqn", "xbeta")
    pin = {k: x[k].pin_memory() for k in names}
    hout = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    dbuf = dict(d)
    for k in names:
        dbuf[k] = torch.empty_like(d[k])
    e_t, e_steps = 0.0, max(3, min(args.e2e_steps, args.steps))
    for i in range(e_steps + 2):
        flush.fill_(1)
        sweep.sum()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for k in names:
            dbuf[k].copy_(pin[k], non_blocking=True)
        kla.prologue(**dbuf, cu_seqlens=cu, B=None if cu is not None else w.B, T=None if cu is not None else w.T,
                     mode=w.mode, out=outs)
        for ho, o in zip(hout, outs):
            ho.copy_(o, non_blocking=True)
        a1.record(stream)
        a1.synchronize()
        if i >= 2:
            e_t += a0.elapsed_time(a1)
    e2e = {"value": w.tokens / (e_t / e_steps * 1e-3), "unit": UNIT,
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pin.values()),
           "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout)}
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    alg = prologue_bytes_per_token_head(w) * w.tokens * H
    ach = alg / (ms * 1e-3) / 1e9
    cfg = arm_config(w, 1)
    cfg["variant"] = "prologue (conv width 4, with bias)"
    res = {"metric": PRO_METRIC, "value": w.tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": cfg,
           "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                        "traffic": None, "kernel": "prologue_kernel", "alg_bytes_per_launch": alg, "launch_ms": ms,
                        "alg_bytes_per_token_head": prologue_bytes_per_token_head(w),
                        "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_src},
           "e2e": e2e, "gpu_launches": args.steps, "clocks": clk}
    if not args.no_cpu_baseline:
        import oracle
        cu_h = inp["cu_seqlens"]
        xs, bounds = _prologue_sample(x, cu_h, w, min(256, Ntok))
        t1 = time.perf_counter()
        oracle.prologue(**xs, cu_seqlens=bounds)
        per_tok = max(time.perf_counter() - t1, 1e-4) / min(256, Ntok)
        n = int(max(1, min(Ntok, 8192, 12.0 / per_tok)))
        xs, bounds = _prologue_sample(x, cu_h, w, n)
        t0 = time.perf_counter()
        ref = oracle.prologue(**xs, cu_seqlens=bounds)
        t = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": n / t, "unit": UNIT, "cores": 1, "kind": "oracle",
                               "sample": "the first %d of %d tokens (all %d heads), numpy fp64 oracle, %.3f s" % (
                                   n, Ntok, H, t)}
        worst = {}
        for name, o in zip(("q", "k", "v", "a", "qn", "beta"), outs):
            worst[name] = scaled_err(o[:n], ref[name])
        res["max_err"] = dict(worst, tokens=n, tol=2e-2 if w.dtype == "bf16" else 1e-4,
                              definition="max |gpu - oracle| / (1 + |oracle|) over the sampled tokens")
    print(json.dumps(res))


BWD_METRIC = "KLA backward (all input gradients) tokens/s per layer (B*T/s) on 1 B200; % of HBM"


def backward_bytes_per_token_head(w) -> int:
    """Algorithmic bytes of the backward per (token, head): the forward's
    inputs and dL/dout read once, every gradient written once (fp32)."""
    es = 2 if w.dtype == "bf16" else 4
    nl = 1 if w.mode == "iso" else w.dk
    return es * (2 * w.dk + 2 * w.dv) + 4 * 2 * nl + 4 + 4 * (2 * w.dk + w.dv + 2 * nl + 1)


def run_backward(args, w):
    """kla_backward on the workload (gradients of every input given a random
    dL/dout): device-timed with L2 flushed between steps against its
    algorithmic bytes; end to end with the inputs and dL/dout copied in from
    pinned host memory and the gradients copied back inside the timed region;
    the fp64 oracle's reverse mode on a few units as the CPU baseline."""
    from bayesian_filter_scan_b200 import kla
    torch.cuda.set_device(0)
    kla.lib()
    inp = make_inputs(w, seed=rank_seed(w, 0))
    g = torch.Generator().manual_seed(w.seed + 1)
    inp["dout"] = torch.randn(inp["v"].shape, generator=g).to(inp["v"].dtype)
    names = ("q", "k", "v", "a", "qn", "beta", "dout")
    dev = {k: inp[k].cuda() for k in names}
    cu = inp["cu_seqlens"].cuda() if inp["cu_seqlens"] is not None else None
    desc, _ = kla._desc_from(dev["q"], dev["v"], w.B, w.T, kla._mode(w.mode), cu)
    ws = torch.empty(max(16, kla.lib().kla_backward_workspace_bytes(ctypes.byref(desc))), dtype=torch.uint8,
                     device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    sweep = torch.ones(SWEEP_BYTES // 4, dtype=torch.float32, device="cuda")

    def run(d):
        return kla.backward(d["q"], d["k"], d["v"], d["a"], d["qn"], d["beta"], d["dout"], cu_seqlens=cu,
                            B=w.B, T=w.T, mode=w.mode, workspace=ws)

    def flush_l2():
        flush.fill_(1)
        sweep.sum()
    for _ in range(args.warmup):
        flush_l2()
        run(dev)
    torch.cuda.synchronize()
    kla.check()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(0)
    clocks.start()
    for e0, e1 in ev:
        flush_l2()
        e0.record(stream)
        grads = run(dev)
        e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    kla.check()
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    # end to end: pinned inputs in, the gradients out, inside the timed region
    pin = {k: inp[k].pin_memory() for k in names}
    hout = {k: torch.empty(t.shape, dtype=t.dtype).pin_memory() for k, t in grads.items()}
    dbuf = {k: torch.empty_like(dev[k]) for k in names}
    e_t, e_steps = 0.0, max(3, min(args.e2e_steps, args.steps))
    for i in range(e_steps + 2):
        flush_l2()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for k in names:
            dbuf[k].copy_(pin[k], non_blocking=True)
        got = run(dbuf)
        for k, t in got.items():
            hout[k].copy_(t, non_blocking=True)
        a1.record(stream)
        a1.synchronize()
        if i >= 2:
            e_t += a0.elapsed_time(a1)
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    alg = backward_bytes_per_token_head(w) * w.tokens * w.H
    ach = alg / (ms * 1e-3) / 1e9
    cfg = arm_config(w, 1)
    cfg["variant"] = "backward (all input gradients, random dL/dout)"
    res = {"metric": BWD_METRIC, "value": w.tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": cfg,
           "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                        "traffic": None, "kernel": "kla_backward (five launches, CUDA cores)",
                        "alg_bytes_per_launch": alg, "launch_ms": ms,
                        "alg_bytes_per_token_head": backward_bytes_per_token_head(w),
                        "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_src},
           "e2e": {"value": w.tokens / (e_t / e_steps * 1e-3), "unit": UNIT,
                   "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pin.values()),
                   "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout.values())},
           "gpu_launches": args.steps * (7 if w.mode == "iso" else 5), "clocks": clk}
    if not args.no_cpu_baseline:
        import oracle
        n_units = min(4, _units_total(w, inp))
        t0 = time.perf_counter()
        ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["a"], inp["qn"], inp["beta"], inp["dout"],
                              cu_seqlens=inp["cu_seqlens"], B=None if inp["cu_seqlens"] is not None else w.B,
                              T=None if inp["cu_seqlens"] is not None else w.T, iso=w.mode == "iso",
                              units=(0, n_units), num_threads=n_units)
        t = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": _unit_tokens(w, inp, n_units) / t, "unit": UNIT, "cores": n_units,
                               "kind": "oracle",
                               "sample": "%d of %d (row, head) units, fp64 C oracle (reverse mode), %.3f s" % (
                                   n_units, _units_total(w, inp), t)}
        cuh = inp["cu_seqlens"].tolist() if inp["cu_seqlens"] is not None else None
        worst = {}
        for name, gt in grads.items():
            gs, ws_ = [], []
            for u in range(n_units):
                n, h = divmod(u, w.H)
                if name in ("dlambda0", "deta0"):
                    gs.append(gt[n, h].reshape(-1))
                    ws_.append(ref[name][n, h].reshape(-1))
                else:
                    s0, s1 = (cuh[n], cuh[n + 1]) if cuh else (n * w.T, (n + 1) * w.T)
                    gs.append(gt[s0:s1, h].reshape(-1))
                    ws_.append(ref[name][s0:s1, h].reshape(-1))
            gv = torch.cat(gs).double().cpu().numpy()
            wv = np.concatenate(ws_)
            scale = float(np.max(np.abs(wv))) if wv.size else 0.0
            worst[name] = float(np.max(np.abs(gv - wv))) / (scale + 1e-30) if wv.size else 0.0
        res["max_err"] = dict(worst, units=n_units, tol=2e-3,
                              definition="max |gpu - oracle| / max |oracle| per gradient over the sampled units")
    print(json.dumps(res))


def run_reference(args, w):
    """Reference arm: the CPU oracle timed on this host's cores. It loads only
    the oracle, never the CUDA library."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    inp = make_inputs(w)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_units = sample_units(w, inp, budget)
    for _ in range(args.warmup):
        oracle.forward_inputs(inp, w, units=(0, n_units), want_final=False)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward_inputs(inp, w, units=(0, n_units), want_final=False)
        ts.append(time.perf_counter() - t0)
    t = sum(ts) / len(ts)
    value = _unit_tokens(w, inp, n_units) / t
    sample = "%d of %d (row, head) units per step, fp64 C oracle" % (n_units, _units_total(w, inp))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", default="kla", choices=["kla", "kdn", "prologue", "backward"],
                    help="kla: the KLA forward (the bench line); kdn: the Kalman Delta Network "
                         "residual write on the same workload; prologue: the mixer's input "
                         "prologue; backward: the gradients of the KLA forward (separate lines)")
    ap.add_argument("--T", type=int, default=None,
                    help="tokens per row instead of the workload's (smaller cases of the same "
                         "workload for profiler captures; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.T is not None:
        w = w.with_(T=args.T)
    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.variant == "kdn":
        run_kdn(args, w)
        return
    if args.variant == "prologue":
        run_prologue(args, w)
        return
    if args.variant == "backward":
        run_backward(args, w)
        return

    from bayesian_filter_scan_b200 import kla

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    kla.lib()
    inp = make_inputs(w, seed=rank_seed(w, rank))
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    Ntok = w.tokens
    H, dk, dv = w.H, w.dk, w.dv
    cu = dev["cu_seqlens"]
    N = cu.numel() - 1 if cu is not None else w.B
    mode = kla.KLA_ISO if w.mode == "iso" else kla.KLA_DIAG
    dt = kla.KLA_BF16 if w.dtype == "bf16" else kla.KLA_FP32
    desc = kla.make_desc(w.B, w.T, H, dk, dv, dt, mode, cu, N if cu is not None else 0)
    plan = kla.plan(desc)
    out = torch.empty(Ntok, H, dv, dtype=dev["q"].dtype, device="cuda")
    fl = torch.empty((N, H) if mode == kla.KLA_ISO else (N, H, dk), device="cuda") if w.final_state else None
    fe = torch.empty(N, H, dk, dv, device="cuda") if w.final_state else None
    nws = kla.workspace_bytes(desc)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    sweep = torch.ones(SWEEP_BYTES // 4, dtype=torch.float32, device="cuda")

    def flush_l2():
        # write 512 MiB (evicts every line of ours), then read 256 MiB so that the
        # flush's own dirty lines are written back here, not inside the timed step
        flush.fill_(1)
        sweep.sum()
    stream = torch.cuda.current_stream()
    L = kla.lib()
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    args_fwd = [ctypes.byref(desc), P(dev["q"]), P(dev["k"]), P(dev["v"]), P(dev["a"]), P(dev["qn"]),
                P(dev["beta"]), P(dev["lambda0"]), P(dev["eta0"]), P(out), P(fl), P(fe), P(ws), nws,
                ctypes.c_void_p(stream.cuda_stream)]

    steps = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
    for row in evs:
        for e in row:
            e.record(stream)   # materialise the events
    torch.cuda.synchronize()
    ev_ptrs = [(ctypes.c_void_p * 7)(*[ctypes.c_void_p(e.cuda_event) for e in row]) for row in evs]

    # timed steps: one kla_forward between two events (the headline); the
    # per-launch breakdown comes from a separate run with an event between
    # every launch, whose extra records would otherwise sit inside the timing
    fwd_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]

    def step(i=None, profiled=False):
        flush_l2()
        if profiled:
            s = L.kla_forward_profiled(*args_fwd, ev_ptrs[i])
        else:
            if i is not None:
                fwd_ev[i][0].record(stream)
            s = L.kla_forward(*args_fwd)
            if i is not None:
                fwd_ev[i][1].record(stream)
        if s != kla.KLA_OK:
            raise kla.KlaError(s, "kla_forward")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    kla.check()
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    t_wall = time.perf_counter()
    for i in range(steps):
        step(i)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    barrier()
    kla.check()
    tot = [e0.elapsed_time(e1) for e0, e1 in fwd_ev]         # ms, whole forward
    for i in range(steps):
        step(i, profiled=True)
    torch.cuda.synchronize()
    kla.check()
    walk = [r[4].elapsed_time(r[5]) for r in evs]             # ms, the walk kernel
    pre = [r[0].elapsed_time(r[4]) for r in evs]
    reduce_ms = statistics.mean(r[0].elapsed_time(r[1]) for r in evs)
    # the launches of this plan, by the event pair that brackets each (an event
    # between every launch; stages without a launch of this plan are left out)
    if plan["tensor_core"] and plan["segments"] > 1:
        named = [(0, "mobius_reduce")] + ([(1, "mobius_carry")] if plan["launches"] == 5 else []) + \
                [(4, "segment_walk"), (5, "segment_starts_and_correction")]
        walk_label = "kla_chunk_tc_kernel (segment walk)"
    elif plan["segments"] > 1:
        named = [(0, "mobius_reduce"), (1, "mobius_carry"), (2, "state_pass"), (3, "state_carry"), (4, "output_pass")]
        walk_label = "kla_walk_simt (output pass)"
    else:
        named = ([(0, "sequence_order")] if plan["launches"] == 2 else []) + [(4, "walk")]
        walk_label = "kla_chunk_tc_kernel (whole rows)" if plan["tensor_core"] else "kla_walk_simt"
    per_stage = {n: statistics.mean(r[i].elapsed_time(r[i + 1]) for r in evs) for i, n in named}
    ms_per_step, value = aggregate(world, w.tokens, sum(tot), steps, dist)

    # ---- e2e through the host-buffer entry point
    pin = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    hdesc = kla.make_desc(w.B, w.T, H, dk, dv, dt, mode, None, N if cu is not None else 0)
    if cu is not None:
        hdesc.cu_seqlens = ctypes.c_void_p(pin["cu_seqlens"].data_ptr())
    hout = torch.empty(Ntok, H, dv, dtype=inp["q"].dtype).pin_memory()
    nb = L.kla_host_device_bytes(ctypes.byref(hdesc))
    dbuf = torch.empty(nb, dtype=torch.uint8, device="cuda")
    h_in = sum(t.numel() * t.element_size() for k_, t in pin.items()
               if t is not None and k_ in ("q", "k", "v", "a", "qn", "beta", "cu_seqlens"))
    h_out = hout.numel() * hout.element_size()
    hargs = [ctypes.byref(hdesc), P(pin["q"]), P(pin["k"]), P(pin["v"]), P(pin["a"]), P(pin["qn"]),
             P(pin["beta"]), None, None, P(hout), None, None, P(dbuf), nb, ctypes.c_void_p(stream.cuda_stream)]
    e2e_steps = max(3, min(args.e2e_steps, steps))
    for _ in range(3):
        flush_l2()
        kla._check(L.kla_forward_host(*hargs), "kla_forward_host")
    e_t = 0.0
    for _ in range(e2e_steps):
        flush_l2()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        kla._check(L.kla_forward_host(*hargs), "kla_forward_host")
        a1.record(stream)
        a1.synchronize()
        e_t += a0.elapsed_time(a1)
    _, e2e_value = aggregate(world, w.tokens, e_t, e2e_steps, dist)
    del pin, hout, dbuf
    if dist is not None:
        dist.destroy_process_group()

    if rank != 0:
        return
    peaks, peak_src = measured_peaks()
    units = w.tokens * H
    alg_bytes = bytes_per_token_head(w) * units
    walk_ms = statistics.mean(walk)
    achieved = alg_bytes / (walk_ms * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    # the committed DRAM record is of the workload's own size
    traffic = traffic_record(args.workload) if not args.T else None
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": arm_config(w, world),
        "plan": {"segments_per_row": plan["segments"], "launches_per_step": plan["launches"],
                 "tensor_core_chunk_kernel": plan["tensor_core"]},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": walk_label,
                     "alg_bytes_per_launch": alg_bytes, "launch_ms": walk_ms,
                     "alg_bytes_per_token_head": bytes_per_token_head(w),
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_src},
        "stages_ms": {"note": "separate run with an event between every launch (each adds about 2.6 us)",
                      "before_walk": statistics.mean(pre), "walk_kernel": walk_ms,
                      "total": statistics.mean(r[0].elapsed_time(r[6]) for r in evs), "launches": per_stage},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h_in, "d2h_bytes_per_step": h_out},
        "gpu_launches": steps * plan["launches"],
        "clocks": clk,
        "timed_region_wall_s": t_wall,
    }
    if plan["segments"] > 1 and plan["tensor_core"]:
        sbytes = scan_bytes_per_token_head(w) * units
        sach = sbytes / (reduce_ms * 1e-3) / 1e9
        res["roofline_scan"] = {"bound": "hbm", "kernel": "mobius_reduce_tma (precision scan)",
                                "achieved": sach, "peak": peak, "unit": "GB/s", "frac": sach / peak,
                                "alg_bytes_per_launch": sbytes, "launch_ms": reduce_ms,
                                "alg_bytes_per_token_head": scan_bytes_per_token_head(w)}
    if world == 1 and not args.no_cpu_baseline:
        rec, ref, n_units = cpu_baseline(w, inp)
        res["cpu_baseline"] = rec
        res["max_err"] = max_err(w, inp, ref, n_units, out, fl, fe)
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
