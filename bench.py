#!/usr/bin/env python
"""Benchmark of the B200 selective scan (one JSON line on rank 0).

A step is one ssm_scan_fwd call (carry pass + main pass) over one batch of the
synthetic Mamba-shaped workload, inputs resident in HBM, L2 flushed (256 MB
write) before every timed step, each step timed with CUDA events on the
launching stream. With torchrun (N > 1) every rank scans its own batch shard
of an N-times larger global batch (weak scaling, no data-path collective);
the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --pass bwd [--workload NAME]  # the backward pass (gradients)
  python bench.py --op conv [--workload NAME]   # the block's causal conv1d + SiLU
  python bench.py --op ssd [--workload NAME]    # the multi-head SSD scan (Mamba-2)
  python bench.py --impl reference ...   # the fp64 CPU oracle on host cores
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ssm_inputs as gen  # noqa: E402

METRIC = "selective-scan elements/s (B·L·D) and achieved HBM GB/s as % of B200 peak"
DEFAULT_WORKLOAD = "mamba130m_layer_b8_l2048_d1536"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
B200_SMS, FP32_LANES_PER_SM, B200_MAX_SM_MHZ = 148, 128, 1965.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(gen.SCAN_WORKLOADS) + sorted(gen.DECODE_WORKLOADS) +
                    sorted(gen.SSD_WORKLOADS) + sorted(gen.SSD_DECODE_WORKLOADS))
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time ssm_scan_bwd (the gradients) on the same workload")
    ap.add_argument("--learned-a", action="store_true",
                    help="A with no (n+1) A[d,0] structure (as after training): the "
                         "one-exp-per-state path")
    ap.add_argument("--zoh", action="store_true",
                    help="scan with the exact zero-order-hold input term (ssm_scan_fwd_zoh)")
    ap.add_argument("--op", default="scan", choices=["scan", "conv", "ssd"],
                    help="conv: time the block's causal conv1d + SiLU (forward and backward) "
                         "on the workload's (batch, seqlen, dim); ssd: the multi-head SSD scan "
                         "(default workload " + "ssd_mamba2_b4_l4096_h64_p64_n128)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip timing the other scan workloads and the decode workload")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def algorithmic_bytes(w, batch):
    """Bytes a scan must move at least: inputs read once, outputs written
    once, no (B, L, D, N) intermediates."""
    es = 2 if w.io == "bf16" else 4
    bld, bln = batch * w.seqlen * w.dim, batch * w.seqlen * w.dstate
    per_elem = (4 if w.gate else 3) * es  # x, delta, (z), y
    state = batch * w.dim * w.dstate * 4 * (2 if w.with_h0 else 1)  # h_last (+ h0)
    params = w.dim * w.dstate * 4 + w.dim * 4 * (2 if w.skip else 1)  # A, bias, (D)
    return bld * per_elem + 2 * bln * es + state + params


def alu_ops_per_element(w, zoh=False):
    """FP32 operations the recurrence needs per element in its plain form:
    per state one multiply for the decay power, one for Delta x B, one FMA for
    the state and one for the readout (4N), as counted for the roofline. The
    exact ZOH input term adds one operation per state (the power
    exp(Delta A_n) - 1 next to the decay): 5N."""
    return (5 if zoh else 4) * w.dstate


def measured_traffic(workload, record="traffic.json"):
    """DRAM bytes per call from the committed ncu capture (profiles/<record>),
    or None when the kernel sources changed since that capture (or none was
    taken)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", record)) as f:
            t = json.load(f)
        h = hashlib.sha256()
        for src in t["kernel_sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != t["kernel_sources_sha256"]:
            return None
        return t["workloads"].get(workload, {}).get("per_call")
    except Exception:
        return None


FALLBACK_BF16_TFLOPS = 1590.0


def measured_bf16_peak():
    """Dense bf16 tensor peak: the burst figure (a kernel timed alone)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, interval_s=0.0002):
        self.samples, self.reasons, self.max_mhz, self.error = [], 0, None, None
        self.interval = interval_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            idx = device_index
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                idx = int(vis.split(",")[device_index])
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            # the first queries are slow (lazy set-up): made here, outside the
            # timed region, so that sampling starts at once
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            get_reasons(self.h)
        except Exception as e:  # pragma: no cover - depends on the machine
            self.nvml, self.error = None, f"nvml unavailable: {e}"
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        get_reasons = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception as e:  # pragma: no cover
                self.error = str(e)
                return
            time.sleep(self.interval)

    def __enter__(self):
        # the main thread holds the GIL while it enqueues launches; a short
        # switch interval lets this thread take a sample every interval
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(min(self._switch, self.interval / 2))
        if self.nvml:
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nvml:
            self.t.join()
        sys.setswitchinterval(self._switch)

    def summary(self):
        if not self.nvml:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def cpu_oracle_rate(w, inp, target_s, rng_seed=0, zoh=False):
    """Oracle throughput (elements/s) on a bounded sample of the workload's
    channels, all host threads. Returns (value, cores, sample text)."""
    import oracle
    threads = gen.default_threads()
    batch = inp["x"].shape[0]
    rng = np.random.default_rng(rng_seed)
    all_ch = [(b, d) for b in range(batch) for d in range(w.dim)]

    def run(n):
        idx = rng.choice(len(all_ch), size=min(n, len(all_ch)), replace=False)
        chans = [all_ch[i] for i in idx]
        t0 = time.perf_counter()
        oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                              z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"], io=w.io,
                              channels=chans, nthreads=threads, zoh=zoh)
        return len(chans), time.perf_counter() - t0

    n, dt = run(threads)  # calibration
    per_chan = dt / max(n, 1) * threads
    n2 = int(max(threads, min(len(all_ch), target_s / max(per_chan, 1e-9) * threads)))
    n2 = max(threads, n2 // threads * threads)
    n, dt = run(n2)
    # the whole workload in well under the target: time repeated passes of it
    passes = 1
    if n == len(all_ch) and dt < target_s / 2:
        extra = min(99, int(np.ceil(target_s / max(dt, 1e-9))) - 1)
        for _ in range(extra):
            dt += run(n2)[1]
        passes += extra
    value = passes * n * w.seqlen / dt
    rep = f", {passes} passes" if passes > 1 else ""
    return value, threads, f"{n} of {len(all_ch)} channels x {w.seqlen} steps{rep}, {dt:.1f} s"


# Workloads reported beside the bench workload in `per_config` (one GPU).
PER_CONFIG_SCANS = ("mamba130m_layer_b8_l2048_d1536", "pythia1b_layer_b4_l4096_d4096_h0",
                    "long_b1_l262144_d1536")
PER_CONFIG_DECODE = "decode_b128_d4096_x1000"


SCAN_BATCHED_INPUTS = ("x", "delta", "z", "B", "C", "h0")


def pipelined_host_step(pinned, d, y, h_last, y_host, h_host, step_rows, nb, nch, streams):
    """One end-to-end scan step from pinned host inputs to pinned host results,
    enqueued on the current stream and two copy streams: the batch goes
    through in `nch` row chunks, so the copy of chunk j+1 in, the scan of
    chunk j and the copy of chunk j-1 out overlap (PCIe carries both
    directions at once). Every byte of the step's inputs and results crosses.
    Returns with the current stream waiting on the last copy out."""
    import torch

    s_in, s_out = streams
    cur = torch.cuda.current_stream()
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    bounds = [(nb * j // nch, nb * (j + 1) // nch) for j in range(nch)]
    for j, (r0, r1) in enumerate(bounds):
        with torch.cuda.stream(s_in):
            for k, t in pinned.items():
                if t is None:
                    continue
                if k in SCAN_BATCHED_INPUTS:
                    d[k][r0:r1].copy_(t[r0:r1], non_blocking=True)
                elif j == 0:
                    d[k].copy_(t, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
        cur.wait_event(ev_in)
        step_rows(r0, r1)
        ev_c = torch.cuda.Event()
        ev_c.record(cur)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c)
            y_host[r0:r1].copy_(y[r0:r1], non_blocking=True)
            h_host[r0:r1].copy_(h_last[r0:r1], non_blocking=True)
    cur.wait_stream(s_out)


def time_scan(w, nb, b0, device, K, warmup, zoh=False, learned_a=False, sync=None,
              sample_clocks=False):
    """K timed ssm_scan_fwd calls of workload `w` (batch rows b0 .. b0+nb of its
    global batch) on `device`: inputs resident in HBM, the L2 flushed (256 MB
    write) before every call, each call between CUDA events on the launching
    stream. Returns the per-call times and what the caller needs to reuse the
    call (inputs on the host and device, outputs, the plan, the call)."""
    import torch

    from selective_state_space_39_b200 import scan_plan, scan_workspace_bytes, ssm_scan_fwd

    inp = gen.workload_inputs(w, batch=nb, batch_offset=b0)
    if learned_a:
        inp["A"] = gen.a_matrix_learned(w.dim, w.dstate, w.seed)
    dtype = torch.bfloat16 if w.io == "bf16" else torch.float32

    def to_dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    d = {k: to_dev(v) for k, v in inp.items()}
    y = torch.empty((nb, w.seqlen, w.dim), dtype=dtype, device=device)
    h_last = torch.empty((nb, w.dim, w.dstate), dtype=torch.float32, device=device)
    ws = torch.empty(max(1, scan_workspace_bytes(nb, w.seqlen, w.dim, w.dstate, dtype)),
                     dtype=torch.uint8, device=device)
    plan = scan_plan(nb, w.seqlen, w.dim, w.dstate, dtype)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def step():
        ssm_scan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                     delta_bias=d["delta_bias"], h0=d["h0"], y=y, h_last=h_last, workspace=ws,
                     zoh=zoh)

    def step_rows(r0, r1):
        """The same call on batch rows r0 .. r1 (rows are independent)."""
        rows = lambda t: None if t is None else t[r0:r1]
        ssm_scan_fwd(rows(d["x"]), rows(d["delta"]), d["A"], rows(d["B"]), rows(d["C"]),
                     D=d["D"], z=rows(d["z"]), delta_bias=d["delta_bias"], h0=rows(d["h0"]),
                     y=y[r0:r1], h_last=h_last[r0:r1], workspace=ws, zoh=zoh)

    for _ in range(max(3, warmup)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(device.index) if sample_clocks else None
    if sync:
        sync()
    torch.cuda.synchronize()
    if sampler:
        sampler.__enter__()
    for i in range(K):
        flush.fill_(i & 0xFF)
        starts[i].record()
        step()
        ends[i].record()
    torch.cuda.synchronize()
    if sampler:
        sampler.__exit__(None, None, None)
    if sync:
        sync()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return {"step_ms": step_ms, "plan": plan, "inp": inp, "d": d, "y": y, "h_last": h_last,
            "step": step, "step_rows": step_rows,
            "clocks": sampler.summary() if sampler else None}


def scan_rooflines(w, nb, mean_s, clocks, zoh, plan, traffic):
    """The call's HBM roofline (the workload metric: algorithmic bytes of the
    call over its mean time, against the measured copy bandwidth) and its FP32
    ALU figure (4N operations per element against 148 SMs x 128 lanes at the
    sampled SM clock)."""
    kernel = "%s: carry pass + main pass (%d launches)" % (
        "ssm_scan_fwd_zoh" if zoh else "ssm_scan_fwd", plan.kernels)
    peak, peak_kind = measured_hbm_peak()
    algo = algorithmic_bytes(w, nb)
    achieved = algo / mean_s / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel,
                "algorithmic_bytes_per_launch": algo, "peak_kind": peak_kind}
    sm_mhz = (clocks or {}).get("sm_mhz") or B200_MAX_SM_MHZ
    alu_peak = B200_SMS * FP32_LANES_PER_SM * sm_mhz * 1e6 / 1e9  # Gop/s
    alu = alu_ops_per_element(w, zoh) * nb * w.seqlen * w.dim / mean_s / 1e9
    alu_roofline = {"bound": "alu", "achieved": round(alu, 1), "peak": round(alu_peak, 1),
                    "unit": "Gop/s", "frac": round(alu / alu_peak, 4),
                    "ops_per_element": alu_ops_per_element(w, zoh),
                    "peak_kind": f"derived: {B200_SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                                 f"{sm_mhz:.0f} MHz sampled SM clock"}
    return roofline, alu_roofline


def scan_summary(w, run, traffic):
    """One `per_config` entry for a scan workload."""
    mean_s = statistics.mean(run["step_ms"]) * 1e-3
    roof, alu = scan_rooflines(w, w.batch, mean_s, run["clocks"], False, run["plan"], traffic)
    return {"metric": METRIC, "value": w.batch * w.seqlen * w.dim / mean_s,
            "unit": "elements/s", "ms_per_step": mean_s * 1e3, "steps": len(run["step_ms"]),
            "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
                       "dstate": w.dstate, "io": w.io, "h0": w.with_h0,
                       "segments": run["plan"].segments,
                       "l2": "flushed (256 MB write) before every timed step"},
            "roofline": roof, "alu_roofline": alu, "clocks": run["clocks"]}


def time_decode(w, device, K, warmup):
    """ssm_state_update calls of decode workload `w` on a resident fp32 state
    (one step = one call over all batch rows and channels), timed four ways:
    L2 flushed by a 256 MB write before every call, flushed by a 256 MB read,
    back to back, and the workload's whole run of w.steps calls captured in
    one CUDA graph. Returns the per-call times in ms and the clock record."""
    import torch

    from selective_state_space_39_b200 import ssm_state_update
    dtype = torch.bfloat16 if w.io == "bf16" else torch.float32
    const = gen.decode_constants(w.dim, w.dstate, w.seed)

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    steps_in = [{k: to_dev(v) for k, v in gen.make_decode_inputs(
        w.batch, w.dim, w.dstate, w.io, w.seed, i).items()} for i in range(8)]
    A, D, bias = (to_dev(const[k]) for k in ("A", "D", "delta_bias"))
    state = torch.zeros((w.batch, w.dim, w.dstate), dtype=torch.float32, device=device)
    y = torch.empty((w.batch, w.dim), dtype=dtype, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def call(i):
        s = steps_in[i % len(steps_in)]
        ssm_state_update(state, s["x"], s["delta"], A, s["B"], s["C"], D=D, z=s["z"],
                         delta_bias=bias, y=y)

    for i in range(max(3, warmup)):
        call(i)
    torch.cuda.synchronize()

    # A decode call is short on the GPU and longer than that on the host
    # (Python, argument checks, the launch), so before each timed call the
    # stream is held by a GPU-side delay (outside the events): the call is
    # enqueued before the stream reaches it, and the events time the device.
    def hold(n=1):
        torch.cuda._sleep(200_000 * n)

    def timed(prep, fn=call):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for i in range(K):
            prep(i)
            hold()
            ev[i][0].record()
            fn(i)
            ev[i][1].record()
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    # (1) write-flushed: the call also pays for writing back the flush's dirty
    #     lines; (2) read-flushed (clean lines): the call's own DRAM traffic;
    #     (3) back to back: the 33.5 MB state stays in L2, as across
    #     consecutive decode steps; (4) one CUDA graph of w.steps calls.
    sampler = ClockSampler(device.index)
    with sampler:
        cold_ms = timed(lambda i: flush.fill_(i & 0xFF))
    read_ms = timed(lambda i: flush.view(torch.int64).sum())
    # the stream floor for the state's bytes: torch's device copy of the fp32
    # state (read once, written once), timed the same way (a library kernel,
    # outside the decode path)
    state2 = torch.empty_like(state)
    copy_ms = timed(lambda i: flush.view(torch.int64).sum(), fn=lambda i: state2.copy_(state))
    del state2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold(K)  # every call is enqueued before the stream reaches e0
    e0.record()
    for i in range(K):
        call(i)
    e1.record()
    torch.cuda.synchronize()
    warm_ms = e0.elapsed_time(e1) / K
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(0)  # first call outside capture (library state, attributes)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(w.steps):
            call(i)
    g.replay()  # warm the graph
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record()
    g.replay()
    g1.record()
    torch.cuda.synchronize()
    graph_ms = g0.elapsed_time(g1) / w.steps
    del g
    return {"w": w, "K": K, "cold_ms": cold_ms, "read_ms": read_ms, "warm_ms": warm_ms,
            "graph_ms": graph_ms, "copy_ms": copy_ms, "state_bytes": state.numel() * 4,
            "clocks": sampler.summary()}


def decode_algorithmic_bytes(w):
    es = 2 if w.io == "bf16" else 4
    nbd = w.batch * w.dim
    return (nbd * w.dstate * 4 * 2 + nbd * es * 4 + 2 * w.batch * w.dstate * es +
            w.dim * w.dstate * 4 + 2 * w.dim * 4)


def decode_summary(r):
    """The decode step's figures: the read-flushed call is the headline (the
    call's own DRAM traffic); the others beside it."""
    w = r["w"]
    nbd = w.batch * w.dim
    algo = decode_algorithmic_bytes(w)
    peak, peak_kind = measured_hbm_peak()

    def fig(ms):
        gbs = algo / (ms * 1e-3) / 1e9
        return {"ms_per_step": ms, "value": nbd / (ms * 1e-3), "algorithmic_gbs": round(gbs, 1),
                "frac": round(gbs / peak, 4)}

    read_gbs = algo / (r["read_ms"] * 1e-3) / 1e9
    return {"metric": "decode state-update elements/s (B·D per step) and HBM GB/s",
            "value": nbd / (r["read_ms"] * 1e-3), "unit": "elements/s",
            "ms_per_step": r["read_ms"], "steps": r["K"],
            "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "dstate": w.dstate,
                       "io": w.io, "l2": "flushed (256 MB read) before every timed call"},
            "roofline": {"bound": "hbm", "achieved": round(read_gbs, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(read_gbs / peak, 4),
                         "algorithmic_bytes_per_launch": algo, "peak_kind": peak_kind},
            "write_flushed_l2": fig(r["cold_ms"]), "warm_l2": fig(r["warm_ms"]),
            "cuda_graph": dict(fig(r["graph_ms"]), calls=w.steps),
            "state_copy_read_flushed": {
                "ms": r["copy_ms"], "bytes": 2 * r["state_bytes"],
                "gbs": round(2 * r["state_bytes"] / (r["copy_ms"] * 1e-3) / 1e9, 1),
                "what": "torch device copy of the fp32 state (read and written once), L2 "
                        "flushed by a 256 MB read: a stream of the state's bytes alone"},
            "clocks": r["clocks"]}



def reference_arm(args):
    """--impl reference: the fp64 oracle on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return 0
    import oracle
    w = gen.SCAN_WORKLOADS[args.workload]
    threads = gen.default_threads()
    inp = gen.workload_inputs(w)
    rng = np.random.default_rng(1)
    per_step = threads  # channels per step: one per host thread
    all_ch = [(b, d) for b in range(w.batch) for d in range(w.dim)]
    times = []
    for i in range(args.warmup + args.steps):
        idx = rng.choice(len(all_ch), size=per_step, replace=False)
        t0 = time.perf_counter()
        oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                              z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"], io=w.io,
                              channels=[all_ch[j] for j in idx], nthreads=threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps * per_step * w.seqlen / total
    sample = f"{per_step} random channels x {w.seqlen} steps per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "elements/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
                   "dstate": w.dstate, "io": w.io},
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def decode_bench(args):
    """--workload decode_*: ssm_state_update calls on a resident fp32 state
    (one step = one call over all batch rows and channels), timed with the L2
    flushed before every call (write and read flush), back to back (the state
    fits in L2) and in one CUDA graph."""
    import torch
    w = gen.DECODE_WORKLOADS[args.workload]
    r = time_decode(w, torch.device("cuda", 0), args.steps, args.warmup)
    s = decode_summary(r)
    line = {
        "metric": s["metric"], "value": s["value"], "unit": "elements/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": s["ms_per_step"],
        "higher_is_better": True, "dtype": w.io,
        "data": "synthetic (seeded Philox4x32-10, Mamba-shaped recipe)",
        "config": s["config"], "roofline": s["roofline"],
        "write_flushed_l2": s["write_flushed_l2"], "warm_l2": s["warm_l2"],
        "cuda_graph": s["cuda_graph"], "state_copy_read_flushed": s["state_copy_read_flushed"],
        "gpu_launches": 3 * args.steps + w.steps, "clocks": s["clocks"],
    }
    print(json.dumps(line), flush=True)
    return 0


BWD_METRIC = "selective-scan backward elements/s (B·L·D, all gradients)"


def bwd_algorithmic_bytes(w, batch):
    """Bytes the backward must move at least: x, delta, (z), dy read and dx,
    ddelta, (dz) written once per element; B, C read and dB, dC (fp32)
    written per (b, t, n); per-channel parameters and their gradients."""
    es = 2 if w.io == "bf16" else 4
    bld, bln = batch * w.seqlen * w.dim, batch * w.seqlen * w.dstate
    per_elem = ((4 if w.gate else 3) + (3 if w.gate else 2)) * es
    state = batch * w.dim * w.dstate * 4 * (3 if w.with_h0 else 2)  # dh_last, dh0 (+ h0)
    params = 2 * (w.dim * w.dstate * 4 + w.dim * 4 * (2 if w.skip else 1))
    return bld * per_elem + bln * (2 * es + 2 * 4) + state + params


def bwd_alu_ops_per_element(w):
    """FP32 operations of the adjoint loop in its plain form, per state: the
    recomputed update (2), the adjoint (2: C g + mu, then a lam), the four
    products and sums of dB, dC, dA and dDelta's A term (2 each: 8): 12N."""
    return 12 * w.dstate


def cpu_oracle_bwd_rate(w, inp, grads, target_s, rng_seed=0):
    """Backward oracle throughput (elements/s) on a bounded channel sample."""
    import oracle
    threads = gen.default_threads()
    batch = inp["x"].shape[0]
    rng = np.random.default_rng(rng_seed)
    all_ch = [(b, d) for b in range(batch) for d in range(w.dim)]

    def run(n):
        idx = rng.choice(len(all_ch), size=min(n, len(all_ch)), replace=False)
        chans = [all_ch[i] for i in idx]
        t0 = time.perf_counter()
        oracle.selective_scan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                  grads["dy"], D=inp["D"], z=inp["z"],
                                  delta_bias=inp["delta_bias"], h0=inp["h0"],
                                  dh_last=grads["dh_last"], io=w.io, channels=chans,
                                  nthreads=threads)
        return len(chans), time.perf_counter() - t0

    n, dt = run(threads)
    per_chan = dt / max(n, 1) * threads
    n2 = int(max(threads, min(len(all_ch), target_s / max(per_chan, 1e-9) * threads)))
    n2 = max(threads, n2 // threads * threads)
    n, dt = run(n2)
    passes = 1
    if n == len(all_ch) and dt < target_s / 2:
        extra = min(99, int(np.ceil(target_s / max(dt, 1e-9))) - 1)
        for _ in range(extra):
            dt += run(n2)[1]
        passes += extra
    rep = f", {passes} passes" if passes > 1 else ""
    return (passes * n * w.seqlen / dt, threads,
            f"{n} of {len(all_ch)} channels x {w.seqlen} steps (gradients of the listed "
            f"channels){rep}, {dt:.1f} s")


def backward_bench(args):
    """--pass bwd: ssm_scan_bwd on the workload (one GPU), timed like the
    forward: L2 flushed (256 MB write) before every call, CUDA events."""
    import torch

    from selective_state_space_39_b200 import scan_bwd_workspace_bytes, ssm_scan_bwd
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--pass bwd runs on one GPU")
    w = gen.SCAN_WORKLOADS[args.workload]
    device = torch.device("cuda", 0)
    dtype = torch.bfloat16 if w.io == "bf16" else torch.float32
    inp = gen.workload_inputs(w)
    if args.learned_a:
        inp["A"] = gen.a_matrix_learned(w.dim, w.dstate, w.seed)
    grads = gen.make_grad_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.io, w.seed)

    def to_dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    d = {k: to_dev(v) for k, v in inp.items()}
    g = {k: to_dev(v) for k, v in grads.items()}
    ws = torch.empty(max(1, scan_bwd_workspace_bytes(w.batch, w.seqlen, w.dim, w.dstate, dtype)),
                     dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def step():
        return ssm_scan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], g["dy"], D=d["D"],
                            z=d["z"], delta_bias=d["delta_bias"], h0=d["h0"],
                            dh_last=g["dh_last"], workspace=ws)

    for _ in range(max(3, args.warmup)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    sampler = ClockSampler(0)
    with sampler:
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = statistics.mean(step_ms)
    elements = w.batch * w.seqlen * w.dim
    clocks = sampler.summary()
    sm_mhz = clocks.get("sm_mhz") or B200_MAX_SM_MHZ
    alu_peak = B200_SMS * FP32_LANES_PER_SM * sm_mhz * 1e6 / 1e9
    alu = bwd_alu_ops_per_element(w) * elements / (ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    algo = bwd_algorithmic_bytes(w, w.batch)
    gbs = algo / (ms * 1e-3) / 1e9
    kernel = "ssm_scan_bwd: carry, compose, main, two reduce kernels (5 launches)"
    cpu = None
    if not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_bwd_rate(w, inp, grads, args.cpu_seconds)
        cpu = {"value": v, "unit": "elements/s", "cores": cores, "kind": "oracle",
               "sample": sample}
    line = {
        "metric": BWD_METRIC, "value": elements / (ms * 1e-3), "unit": "elements/s",
        "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.io == "bf16" else "f32",
        "data": "synthetic (seeded Philox4x32-10, Mamba-shaped recipe; dy, dh_last N(0,1))",
        "config": {"workload": w.name, "pass": "backward", "batch": w.batch, "seqlen": w.seqlen,
                   "dim": w.dim, "dstate": w.dstate, "io": w.io,
                   "A": "learned-like (unstructured)" if args.learned_a else "(n+1) A[d,0]",
                   "l2": "flushed (256 MB write) before every timed step"},
        "roofline": {"bound": "alu", "achieved": round(alu, 1), "peak": round(alu_peak, 1),
                     "unit": "Gop/s", "frac": round(alu / alu_peak, 4), "traffic": None,
                     "kernel": kernel, "ops_per_element": bwd_alu_ops_per_element(w),
                     "peak_kind": f"derived: {B200_SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                                  f"{sm_mhz:.0f} MHz sampled SM clock"},
        "hbm_roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(gbs / peak, 4), "traffic": None,
                         "kernel": kernel, "algorithmic_bytes_per_launch": algo,
                         "peak_kind": peak_kind},
        "cpu_baseline": cpu, "gpu_launches": 5 * K, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


CONV_METRIC = "causal conv1d + SiLU elements/s (B·L·D) and achieved HBM GB/s"


def conv_bench(args):
    """--op conv: ssm_conv1d_silu_fwd and _bwd (width 4) on the workload's
    (batch, seqlen, dim), one GPU, L2 flushed (256 MB write) before every call.
    The line's value is the forward; the backward is reported beside it."""
    import torch

    from selective_state_space_39_b200 import (conv1d_silu_bwd_workspace_bytes,
                                               ssm_conv1d_silu_bwd, ssm_conv1d_silu_fwd)
    w = gen.SCAN_WORKLOADS[args.workload]
    device = torch.device("cuda", 0)
    dtype = torch.bfloat16 if w.io == "bf16" else torch.float32
    width = 4
    c = gen.make_conv_inputs(w.batch, w.seqlen, w.dim, width, w.io, w.seed)

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    d = {k: to_dev(v) for k, v in c.items()}
    out = torch.empty(d["x"].shape, dtype=dtype, device=device)
    ws = torch.empty(max(1, conv1d_silu_bwd_workspace_bytes(w.batch, w.seqlen, w.dim, width,
                                                            dtype)), dtype=torch.uint8,
                     device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def fwd():
        ssm_conv1d_silu_fwd(d["x"], d["w"], d["bias"], out=out)

    def bwd():
        ssm_conv1d_silu_bwd(d["x"], d["w"], d["dout"], d["bias"], workspace=ws)

    def timed(f, K):
        for _ in range(max(3, args.warmup)):
            flush.fill_(1)
            f()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            f()
            ev[i][1].record()
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    K = args.steps
    sampler = ClockSampler(0)
    with sampler:
        f_ms = timed(fwd, K)
        b_ms = timed(bwd, K)
    es = 2 if w.io == "bf16" else 4
    n = w.batch * w.seqlen * w.dim
    params = w.dim * (width + 1) * 4
    f_bytes = 2 * n * es + params                # x read, out written
    b_bytes = 3 * n * es + 3 * params            # x, dout read, dx written; w, dw, dbias
    peak, peak_kind = measured_hbm_peak()
    f_gbs = f_bytes / (f_ms * 1e-3) / 1e9
    b_gbs = b_bytes / (b_ms * 1e-3) / 1e9
    line = {
        "metric": CONV_METRIC, "value": n / (f_ms * 1e-3), "unit": "elements/s", "n_gpus": 1,
        "steps": K, "warmup": args.warmup, "ms_per_step": f_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.io == "bf16" else "f32",
        "data": "synthetic (seeded Philox4x32-10; x, dout N(0,1); taps, bias U[-0.5, 0.5])",
        "config": {"workload": w.name, "op": "causal conv1d + SiLU, width 4", "batch": w.batch,
                   "seqlen": w.seqlen, "dim": w.dim, "io": w.io,
                   "l2": "flushed (256 MB write) before every timed call"},
        "roofline": {"bound": "hbm", "achieved": round(f_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(f_gbs / peak, 4), "traffic": None,
                     "kernel": "conv_fwd_kernel (1 launch)",
                     "algorithmic_bytes_per_launch": f_bytes, "peak_kind": peak_kind},
        "backward": {"ms_per_step": b_ms, "value": n / (b_ms * 1e-3), "unit": "elements/s",
                     "roofline": {"bound": "hbm", "achieved": round(b_gbs, 1), "peak": peak,
                                  "unit": "GB/s", "frac": round(b_gbs / peak, 4),
                                  "kernel": "conv_bwd_kernel + conv_reduce_kernel (2 launches)",
                                  "algorithmic_bytes_per_call": b_bytes}},
        "gpu_launches": 3 * K, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


SSD_METRIC = "SSD scan elements/s (B·L·H·P) with tensor-core TFLOP/s and HBM GB/s"
DEFAULT_SSD_WORKLOAD = "ssd_mamba2_b4_l4096_h64_p64_n128"


def ssd_cost(w, Q=32):
    """Algorithmic bytes and FLOPs of one SSD call. Bytes: x read and y written
    (bf16), B, C, dt read, h0 read and h_last written (fp32). FLOPs: the
    chunked dual form's products per (batch, head, chunk of Q steps): G X over
    the causal half (Q^2 P), C H and the state's (w X)^T B (2 Q N P each), and
    C B^T over the causal half (Q^2 N), once per chunk (B and C are shared by
    the heads). Q is the chunk length of the kernel that runs (128 for the
    tensor-core kernel, 32 for the mma.sync one)."""
    P, N = w.headdim, w.dstate
    tok = w.batch * w.seqlen
    nbytes = 2 * 2 * tok * w.nheads * P + 2 * 2 * tok * N + 2 * tok * w.nheads + \
        4 * w.batch * w.nheads * P * N * (2 if w.with_h0 else 1)
    flops = tok * w.nheads * (Q * P + 4 * N * P) + tok * Q * N
    return nbytes, flops


def cpu_oracle_ssd_rate(w, inp, target_s, rng_seed=0):
    """Oracle throughput (elements/s) on a bounded sample of (batch, head)
    pairs (single host thread). Returns (value, cores, sample text)."""
    import oracle
    rng = np.random.default_rng(rng_seed)
    pairs_all = [(b, h) for b in range(w.batch) for h in range(w.nheads)]

    def run(n):
        idx = rng.choice(len(pairs_all), size=min(n, len(pairs_all)), replace=False)
        t0 = time.perf_counter()
        oracle.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                        dt_bias=inp["dt_bias"], h0=inp["h0"], io=w.io,
                        pairs=[pairs_all[i] for i in idx])
        return len(idx), time.perf_counter() - t0

    n, dt = run(1)
    n2 = int(max(1, min(len(pairs_all), target_s / max(dt, 1e-9))))
    n, dt = run(n2)
    return (n * w.seqlen * w.headdim / dt, 1,
            f"{n} of {len(pairs_all)} (batch, head) pairs x {w.seqlen} steps, {dt:.1f} s")


def ssd_bench(args):
    """--op ssd / --workload ssd_*: the multi-head SSD scan (ssm_ssd_scan_fwd,
    one launch per step), one GPU, L2 flushed (256 MB write) before every
    timed call. e2e: pinned host inputs copied in, y and h_last copied out,
    every step, through the Python entry point."""
    import torch

    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    w = gen.SSD_WORKLOADS[args.workload]
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    inp = gen.ssd_workload_inputs(w)

    def to_host(a):
        if a is None:
            return None
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) \
            if a.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(a))
        return t.pin_memory()

    h = {k: to_host(v) for k, v in inp.items()}
    d = {k: (v.to(device) if v is not None else None) for k, v in h.items()}
    P, N = w.headdim, w.dstate
    y = torch.empty((w.batch, w.seqlen, w.nheads, P), dtype=torch.bfloat16, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def call():
        return ssm_ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                                dt_bias=d["dt_bias"], h0=d["h0"], return_last_state=True, y=y)

    for _ in range(max(3, args.warmup)):
        flush.fill_(1)
        call()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    sampler = ClockSampler(0)
    with sampler:
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            call()
            ev[i][1].record()
        torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)

    # end to end: host -> device inputs, the call, device -> host outputs
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    hl_host = torch.empty((w.batch, w.nheads, P, N), dtype=torch.float32).pin_memory()
    keys = [k for k in ("x", "dt", "B", "C", "h0") if h[k] is not None]
    h2d = sum(h[k].numel() * h[k].element_size() for k in keys)
    d2h = y_host.numel() * 2 + hl_host.numel() * 4
    E = max(3, args.e2e_steps)
    # the batch in row chunks on three streams (copies in, scans, copies out
    # overlap), as for the scan's end-to-end figure
    hl_dev = torch.empty((w.batch, w.nheads, P, N), dtype=torch.float32, device=device)
    nch = min(w.batch, 4)
    bounds = [(w.batch * j // nch, w.batch * (j + 1) // nch) for j in range(nch)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    cur = torch.cuda.current_stream(device)

    def rows(t, r0, r1):
        return None if t is None else t[r0:r1]

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(E):
        s_in.wait_stream(cur)
        s_out.wait_stream(cur)
        for r0, r1 in bounds:
            with torch.cuda.stream(s_in):
                for k in keys:
                    d[k][r0:r1].copy_(h[k][r0:r1], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            cur.wait_event(ev_in)
            ssm_ssd_scan_fwd(rows(d["x"], r0, r1), rows(d["dt"], r0, r1), d["A"],
                             rows(d["B"], r0, r1), rows(d["C"], r0, r1), D=d["D"],
                             dt_bias=d["dt_bias"], h0=rows(d["h0"], r0, r1),
                             y=y[r0:r1], h_last=hl_dev[r0:r1])
            ev_c = torch.cuda.Event()
            ev_c.record(cur)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c)
                y_host[r0:r1].copy_(y[r0:r1], non_blocking=True)
                hl_host[r0:r1].copy_(hl_dev[r0:r1], non_blocking=True)
        cur.wait_stream(s_out)
    e1.record(cur)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / E

    elems = w.elements
    # the tensor-core kernel serves dstate 64 / 128 with an even head count
    tc = N in (64, 128) and w.nheads % 2 == 0 and os.environ.get("SSM_SSD_LEGACY", "0") == "0"
    nbytes, flops = ssd_cost(w, Q=128 if tc else 32)
    hbm_peak, hbm_kind = measured_hbm_peak()
    tc_peak, tc_kind = measured_bf16_peak()
    gbs = nbytes / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    # the roofline bound is the larger of the two floors
    t_hbm, t_tc = nbytes / (hbm_peak * 1e9), flops / (tc_peak * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(gbs / hbm_peak, 4), "peak_kind": hbm_kind}
    else:
        roof = {"bound": "tensor", "achieved": round(tfs, 1), "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(tfs / tc_peak, 4), "peak_kind": tc_kind}
    roof.update({"traffic": measured_traffic(w.name, "ssd_tc_traffic.json" if tc
                                             else "ssd_traffic.json"),
                 "kernel": f"{'ssd_tc_kernel' if tc else 'ssd_fwd_kernel'}<{N}> (1 launch)",
                 "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
                 "tensor": {"achieved_tflops": round(tfs, 1), "peak": tc_peak,
                            "frac": round(tfs / tc_peak, 4), "peak_kind": tc_kind},
                 "hbm": {"achieved_gbs": round(gbs, 1), "peak": hbm_peak,
                         "frac": round(gbs / hbm_peak, 4), "peak_kind": hbm_kind}})
    line = {
        "metric": SSD_METRIC, "value": elems / (ms * 1e-3), "unit": "elements/s", "n_gpus": 1,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox4x32-10; x, B, C N(0,1), dt N(0,0.25), A -U[1,16])",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                   "nheads": w.nheads, "headdim": P, "dstate": N, "io": w.io,
                   "h0": w.with_h0, "l2": "flushed (256 MB write) before every timed call"},
        "roofline": roof,
        "e2e": {"value": elems / (e2e_ms * 1e-3), "unit": "elements/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": K, "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_ssd_rate(w, inp, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "elements/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)
    return 0


def ssd_decode_bench(args):
    """--workload ssd_decode_*: ssm_ssd_state_update calls on a resident fp32
    state (one step = one call over every sequence, head and row). Timed with
    L2 flushed before every call (by a write, and by a read) and back to back."""
    import torch

    from selective_state_space_39_b200 import ssm_ssd_state_update
    w = gen.SSD_DECODE_WORKLOADS[args.workload]
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    const = gen.ssd_constants(w.nheads, w.seed)

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    steps_in = [{k: to_dev(v) for k, v in gen.make_ssd_decode_inputs(
        w.batch, w.nheads, w.headdim, w.dstate, w.io, w.seed, i).items()} for i in range(8)]
    A, D, bias = (to_dev(const[k]) for k in ("A", "D", "dt_bias"))
    state = torch.zeros((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                        device=device)
    dtype = torch.bfloat16 if w.io == "bf16" else torch.float32
    y = torch.empty((w.batch, w.nheads, w.headdim), dtype=dtype, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def call(i):
        s_ = steps_in[i % len(steps_in)]
        ssm_ssd_state_update(state, s_["x"], s_["dt"], A, s_["B"], s_["C"], D=D, dt_bias=bias,
                             y=y)

    for i in range(max(3, args.warmup)):
        call(i)
    torch.cuda.synchronize()
    K = args.steps

    # A decode call is short on the GPU and longer than that on the host
    # (Python, argument checks, the launch), so before each timed call the
    # stream is held by a GPU-side delay (outside the events): the call is
    # enqueued before the stream reaches it, and the events time the device.
    def hold(n=1):
        torch.cuda._sleep(200_000 * n)

    def timed(prep, fn=call):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for i in range(K):
            prep(i)
            hold()
            ev[i][0].record()
            fn(i)
            ev[i][1].record()
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    sampler = ClockSampler(0)
    with sampler:
        cold_ms = timed(lambda i: flush.fill_(i & 0xFF))
    read_ms = timed(lambda i: flush.view(torch.int64).sum())
    # the stream floor for the state's bytes: torch's device copy of the fp32
    # state, timed the same way (a library kernel, outside the decode path)
    state2 = torch.empty_like(state)
    copy_cold_ms = timed(lambda i: flush.fill_(i & 0xFF), fn=lambda i: state2.copy_(state))
    copy_read_ms = timed(lambda i: flush.view(torch.int64).sum(), fn=lambda i: state2.copy_(state))
    del state2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold(K)  # every call is enqueued before the stream reaches e0
    e0.record()
    for i in range(K):
        call(i)
    e1.record()
    torch.cuda.synchronize()
    warm_ms = e0.elapsed_time(e1) / K
    es = 2 if w.io == "bf16" else 4
    rows = w.batch * w.nheads * w.headdim
    algo = rows * w.dstate * 4 * 2 + rows * es * 2 + w.batch * w.nheads * es + \
        2 * w.batch * w.dstate * es + 3 * w.nheads * 4
    peak, peak_kind = measured_hbm_peak()
    gbs = algo / (cold_ms * 1e-3) / 1e9
    line = {
        "metric": "SSD decode state-update rows/s (B·H·P per step) and HBM GB/s",
        "value": rows / (cold_ms * 1e-3), "unit": "rows/s", "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": cold_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.io,
        "data": "synthetic (seeded Philox4x32-10, the SSD recipe)",
        "config": {"workload": w.name, "batch": w.batch, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate,
                   "l2": "flushed (256 MB write) before every timed call"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None,
                     "kernel": f"ssd_decode_kernel<{w.dstate}> (1 launch)",
                     "algorithmic_bytes_per_launch": algo, "peak_kind": peak_kind},
        "read_flushed_l2": {"ms_per_step": read_ms,
                            "algorithmic_gbs": round(algo / (read_ms * 1e-3) / 1e9, 1),
                            "frac": round(algo / (read_ms * 1e-3) / 1e9 / peak, 4)},
        "back_to_back": {"ms_per_step": warm_ms,
                         "algorithmic_gbs": round(algo / (warm_ms * 1e-3) / 1e9, 1)},
        "state_copy": {
            "bytes": 2 * state.numel() * 4, "write_flushed_ms": copy_cold_ms,
            "read_flushed_ms": copy_read_ms,
            "what": "torch device copy of the fp32 state (read and written once), L2 flushed "
                    "the same two ways: a stream of the state's bytes alone"},
        "gpu_launches": 3 * K, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def decode_reference_arm(args):
    """--impl reference on a decode workload: the fp64 oracle's decode step over
    every batch row and channel (or head row) of the workload, one call per
    step, on the host (rank 0 only)."""
    import oracle
    ssd = args.workload in gen.SSD_DECODE_WORKLOADS
    w = (gen.SSD_DECODE_WORKLOADS if ssd else gen.DECODE_WORKLOADS)[args.workload]
    if ssd:
        const = gen.ssd_constants(w.nheads, w.seed)
        state = np.zeros((w.batch, w.nheads, w.headdim, w.dstate))
        rows = w.batch * w.nheads * w.headdim
    else:
        const = gen.decode_constants(w.dim, w.dstate, w.seed)
        state = np.zeros((w.batch, w.dim, w.dstate))
        rows = w.batch * w.dim
    times = []
    for i in range(args.warmup + args.steps):
        if ssd:
            d = gen.make_ssd_decode_inputs(w.batch, w.nheads, w.headdim, w.dstate, w.io, w.seed,
                                           i)
            t0 = time.perf_counter()
            oracle.ssd_state_update(state, d["x"], d["dt"], const["A"], d["B"], d["C"],
                                    D=const["D"], dt_bias=const["dt_bias"], io=w.io)
        else:
            d = gen.make_decode_inputs(w.batch, w.dim, w.dstate, w.io, w.seed, i)
            t0 = time.perf_counter()
            oracle.state_update(state, d["x"], d["delta"], const["A"], d["B"], d["C"],
                                D=const["D"], z=d["z"], delta_bias=const["delta_bias"], io=w.io)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps * rows / total
    unit = "rows/s" if ssd else "elements/s"
    line = {
        "impl": "reference",
        "metric": ("SSD decode state-update rows/s (B·H·P per step) and HBM GB/s" if ssd else
                   "decode state-update elements/s (B·D per step) and HBM GB/s"),
        "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name},
        "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle",
                         "sample": "every row of the workload, one decode step per step"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def ssd_reference_arm(args):
    """--impl reference on an SSD workload: the fp64 oracle, one (batch, head)
    pair per step, on the host (rank 0 only)."""
    import oracle
    w = gen.SSD_WORKLOADS[args.workload]
    inp = gen.ssd_workload_inputs(w)
    rng = np.random.default_rng(1)
    times = []
    for i in range(args.warmup + args.steps):
        pair = (int(rng.integers(w.batch)), int(rng.integers(w.nheads)))
        t0 = time.perf_counter()
        oracle.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                        dt_bias=inp["dt_bias"], h0=inp["h0"], io=w.io, pairs=[pair])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps * w.seqlen * w.headdim / total
    sample = f"1 random (batch, head) pair x {w.seqlen} steps per step"
    line = {
        "impl": "reference", "metric": SSD_METRIC, "value": value, "unit": "elements/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                   "nheads": w.nheads, "headdim": w.headdim, "dstate": w.dstate, "io": w.io},
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.op == "ssd" and args.workload not in gen.SSD_WORKLOADS:
        args.workload = DEFAULT_SSD_WORKLOAD
    if args.impl == "reference":
        if int(os.environ.get("RANK", 0)) != 0:
            return 0
        if args.workload in gen.SSD_WORKLOADS:
            return ssd_reference_arm(args)
        if args.workload in gen.DECODE_WORKLOADS or args.workload in gen.SSD_DECODE_WORKLOADS:
            return decode_reference_arm(args)
        return reference_arm(args)
    single = (args.op == "conv" or args.workload in gen.SSD_WORKLOADS or
              args.workload in gen.DECODE_WORKLOADS or args.workload in gen.SSD_DECODE_WORKLOADS)
    if single and int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("this mode runs on one GPU (the batch-sharded scan runs on N)")
    if args.workload in gen.SSD_WORKLOADS:
        return ssd_bench(args)
    if args.workload in gen.SSD_DECODE_WORKLOADS:
        return ssd_decode_bench(args)
    if args.workload in gen.DECODE_WORKLOADS:
        return decode_bench(args)
    if args.op == "conv":
        return conv_bench(args)
    if args.which == "bwd":
        return backward_bench(args)

    import torch

    from selective_state_space_39_b200 import dist as sdist

    rank, local_rank, world = sdist.env_world()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the scan has no CPU path)")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    sdist.init("nccl")

    w = gen.SCAN_WORKLOADS[args.workload]
    # weak scaling: global batch = world * w.batch; this rank's shard
    b0, nb = sdist.batch_shard(world * w.batch, world, rank)
    run = time_scan(w, nb, b0, device, args.steps, args.warmup, zoh=args.zoh,
                    learned_a=args.learned_a, sync=lambda: sdist.barrier(device),
                    sample_clocks=True)
    step_ms, plan, inp, d, y, h_last, step, step_rows = (run[k] for k in (
        "step_ms", "plan", "inp", "d", "y", "h_last", "step", "step_rows"))
    dtype = y.dtype
    K = args.steps
    local_ms = sum(step_ms)
    total_ms = sdist.max_over_ranks(local_ms, device)
    ms_per_step = total_ms / K
    elements = world * w.batch * w.seqlen * w.dim
    value = elements * K / (total_ms * 1e-3)
    clocks = run["clocks"]
    mean_s = statistics.mean(step_ms) * 1e-3
    use_traffic = (world == 1 or nb == w.batch) and not args.zoh and not args.learned_a
    roofline, alu_roofline = scan_rooflines(w, nb, mean_s, clocks, args.zoh, plan,
                                            measured_traffic(w.name) if use_traffic else None)

    # end to end through the public call: pinned host inputs -> device -> scan -> host
    e2e = None
    if args.e2e_steps > 0:
        pinned = {k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v)
                      .view(dtype if v.dtype == np.uint16 else torch.float32).pin_memory()
                      if v is not None else None) for k, v in inp.items()}
        y_host = torch.empty(y.shape, dtype=dtype).pin_memory()
        h_host = torch.empty(h_last.shape, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
        d2h = y_host.numel() * y_host.element_size() + h_host.numel() * h_host.element_size()
        # 4 chunks measured best on the 8 x 2048 x 1536 layer (3.39 ms a step,
        # against 3.49 with 2 and 3.53 with 8; SSM_BENCH_E2E_CHUNKS sets it).
        nch = max(1, min(nb, int(os.environ.get("SSM_BENCH_E2E_CHUNKS", "4"))))
        streams = (torch.cuda.Stream(device), torch.cuda.Stream(device))
        e_ms = []
        for i in range(args.e2e_steps + 2):
            cur = torch.cuda.current_stream(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(cur)
            pipelined_host_step(pinned, d, y, h_last, y_host, h_host, step_rows, nb, nch,
                                streams)
            e1.record(cur)
            e1.synchronize()
            if i >= 2:
                e_ms.append(e0.elapsed_time(e1))
        e2e_ms = sdist.max_over_ranks(statistics.mean(e_ms), device)
        e2e = {"value": elements / (e2e_ms * 1e-3), "unit": "elements/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "pipeline": f"{nch} batch-row chunks; copies in, scans and copies out overlap"}
    del run, d, y, h_last, step, step_rows

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_rate(w, inp, args.cpu_seconds, zoh=args.zoh)
        cpu = {"value": v, "unit": "elements/s", "cores": cores, "kind": "oracle",
               "sample": sample}
    del inp

    # The other workloads of the scan (and the decode workload), timed the same
    # way in this run on one GPU; they are reported, not part of `value`.
    per_config = None
    if world == 1 and not args.zoh and not args.learned_a and args.per_config:
        per_config = {}
        for name in PER_CONFIG_SCANS:
            if name == w.name:
                continue
            wc = gen.SCAN_WORKLOADS[name]
            rc = time_scan(wc, wc.batch, 0, device, args.steps, args.warmup,
                           sample_clocks=True)
            per_config[name] = scan_summary(wc, rc, measured_traffic(wc.name))
            del rc
            torch.cuda.empty_cache()
        # a decode call is ~20 us: at least 200 timed calls (a few ms in all)
        per_config[PER_CONFIG_DECODE] = decode_summary(
            time_decode(gen.DECODE_WORKLOADS[PER_CONFIG_DECODE], device, max(args.steps, 200),
                        max(args.warmup, 10)))

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.io == "bf16" else "f32",
            "data": "synthetic (seeded Philox4x32-10, Mamba-shaped recipe)",
            "config": {"workload": w.name, "batch_per_gpu": w.batch, "global_batch": world * w.batch,
                       "seqlen": w.seqlen, "dim": w.dim, "dstate": w.dstate, "io": w.io,
                       "gate": w.gate, "skip": w.skip, "h0": w.with_h0,
                       "segments": plan.segments, "segment_steps": plan.segment_steps,
                       "input_term": "exact ZOH" if args.zoh else "Delta B",
                       "A": "learned-like (unstructured)" if args.learned_a else "(n+1) A[d,0]",
                       "l2": "flushed (256 MB write) before every timed step",
                       "parallelism": f"dp{world} (batch shards, no data-path collective)"},
            "hbm_gbs": roofline["achieved"], "hbm_frac_of_peak": roofline["frac"],
            "roofline": roofline, "alu_roofline": alu_roofline, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": K * plan.kernels, "clocks": clocks,
        }
        if per_config is not None:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    sdist.finish()
    return 0


if __name__ == "__main__":
    sys.exit(main())
