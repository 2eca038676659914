#!/usr/bin/env python
"""Throughput benchmark of the Kalman linear-attention forward pass on B200.

One step = one kla_forward call over one batch of the workload (the whole hot
path: Moebius precision scan, state passing, chunked tensor-core pass) with
inputs resident in HBM. Prints ONE JSON line (rank 0):

  value       tokens/s (B*T per second, all ranks together), device-timed with
              CUDA events on the launching stream around each call, L2 flushed
              (512 MiB write) between timed steps, max over ranks;
  e2e         the same metric through kla_forward_host: pinned host inputs
              copied in, forward, output copied back, inside the timed region;
  roofline    the dominant kernel (the chunk kernel walking whole rows, or the
              segments of split rows) against the measured HBM copy bandwidth:
              algorithmic bytes (inputs read once, output written once) / its
              event-timed duration;
  cpu_baseline the CPU oracle (plain fp64 C, OpenMP) on a bounded sample of
              the same workload, on this host's cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1] [--impl reference]

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
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from bayesian_filter_scan_b200 import kla  # noqa: E402
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "KLA forward tokens/s per layer (B*T/s) on 1 B200; % of HBM / bf16 TC roofline"
UNIT = "tokens/s"
FLUSH_BYTES = 512 << 20
SWEEP_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0


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


def flops_per_token_head(w) -> int:
    """The recurrence's own arithmetic: rank-1 state update and readout."""
    return 4 * w.dk * w.dv


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def chunk_kernel_hash() -> str:
    with open(os.path.join(ROOT, "bayesian_filter_scan_b200", "csrc", "kla_chunk_tc.cu"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_record(wid):
    """DRAM bytes per launch of the chunk kernel from a committed ncu summary,
    if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "chunk_kernel_traffic.json")
    try:
        rec = json.load(open(path)).get(str(wid))
    except Exception:
        return None
    if not rec or rec.get("kernel_sha") != chunk_kernel_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="kla_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


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


def cpu_baseline(w, inp, target_s=12.0):
    """The oracle, as it stands, on a bounded sample of (row, head) units."""
    import oracle
    units_total = (inp["cu_seqlens"].numel() - 1 if inp["cu_seqlens"] is not None else w.B) * w.H
    t1 = oracle.time_forward(inp, w, (0, 1))
    per_unit = max(t1, 1e-4)
    n_units = int(max(1, min(units_total, target_s / per_unit * oracle.max_threads())))
    reps, t = 0, 0.0
    while reps == 0 or t < 2.0:       # repeat a small sample for a stable time
        t += oracle.time_forward(inp, w, (0, n_units))
        reps += 1
    t /= reps
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].tolist()
        tok = sum(cu[u // w.H + 1] - cu[u // w.H] for u in range(n_units)) / w.H
    else:
        tok = n_units * w.T / w.H
    return {"value": tok / t, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": "%d of %d (row, head) units of the workload, fp64 C oracle, %.3f s per pass, %d passes" % (
                n_units, units_total, t, reps)}


def arm_config(w, plan, world):
    """The workload's `config` object, the same on both arms."""
    return {"workload": workload_label(w), "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv,
            "mode": w.mode, "varlen": w.varlen, "tokens_per_step_per_gpu": w.tokens,
            "segments_per_row": plan["segments"], "tensor_core_chunk_kernel": plan["tensor_core"],
            "l2": "flushed between timed steps (512 MiB device write, then 256 MiB read)",
            "parallelism": "dp%d" % world}


class _HostOffsets:
    """Stands in for the packed-sequence offsets when only the plan is asked
    for: the plan reads the descriptor's shapes, never the offsets."""

    def data_ptr(self):
        return 256


def host_plan(w, num_seqs):
    mode = kla.KLA_ISO if w.mode == "iso" else kla.KLA_DIAG
    dt = kla.KLA_BF16 if w.dtype == "bf16" else kla.KLA_FP32
    desc = kla.make_desc(w.B, w.T, w.H, w.dk, w.dv, dt, mode, _HostOffsets() if w.varlen else None,
                         num_seqs if w.varlen else 0)
    return kla.plan(desc)


def run_reference(args, w):
    """Reference arm: the CPU oracle timed on this host's cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    inp = make_inputs(w)
    units_total = (inp["cu_seqlens"].numel() - 1 if inp["cu_seqlens"] is not None else w.B) * w.H
    per_unit = max(oracle.time_forward(inp, w, (0, 1)), 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_units = int(max(1, min(units_total, budget / per_unit * oracle.max_threads())))
    for _ in range(args.warmup):
        oracle.time_forward(inp, w, (0, n_units))
    ts = [oracle.time_forward(inp, w, (0, n_units)) for _ in range(args.steps)]
    tok = n_units * w.T / w.H if inp["cu_seqlens"] is None else sum(
        inp["cu_seqlens"][u // w.H + 1].item() - inp["cu_seqlens"][u // w.H].item() for u in range(n_units)) / w.H
    t = sum(ts) / len(ts)
    value = tok / t
    sample = "%d of %d (row, head) units per step, fp64 C oracle" % (n_units, units_total)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(w, host_plan(w, units_total // w.H), args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", type=int, default=1, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    ev_ptrs = [(ctypes.c_void_p * 7)(*[ctypes.c_void_p(e.cuda_event) for e in row]) for row in evs]
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
    clocks = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    clocks.start()
    time.sleep(0.3)
    t_wall = time.perf_counter()
    for i in range(steps):
        step(i)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    barrier()
    clk = clocks.stop()
    kla.check()
    tot = [e0.elapsed_time(e1) for e0, e1 in fwd_ev]         # ms, whole forward
    for i in range(steps):
        step(i, profiled=True)
    torch.cuda.synchronize()
    kla.check()
    chunk = [r[4].elapsed_time(r[5]) for r in evs]            # ms, the walk kernel
    pre = [r[0].elapsed_time(r[4]) for r in evs]
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
    if dist is not None:
        dist.destroy_process_group()

    if rank != 0:
        return
    peaks, peak_src = measured_peaks()
    units = w.tokens * H
    alg_bytes = bytes_per_token_head(w) * units
    chunk_ms = statistics.mean(chunk)
    achieved = alg_bytes / (chunk_ms * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    # the committed DRAM record is of the workload's own size
    traffic = traffic_record(args.workload) if not args.T else None
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": arm_config(w, plan, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": walk_label,
                     "alg_bytes_per_launch": alg_bytes, "launch_ms": chunk_ms,
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_src},
        "stages_ms": {"note": "separate run with an event between every launch (each adds about 2.6 us)",
                      "before_walk": statistics.mean(pre), "walk_kernel": chunk_ms,
                      "total": statistics.mean(r[0].elapsed_time(r[6]) for r in evs), "launches": per_stage},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h_in, "d2h_bytes_per_step": h_out},
        "gpu_launches": steps * plan["launches"],
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                   "samples": clk.get("samples", 0)},
        "timed_region_wall_s": t_wall,
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, inp)
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
