#!/usr/bin/env python
"""Benchmark of the forward selective scan (S6) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one full forward scan (softplus step size, discretisation,
recurrence, C readout, D skip, silu(z) gate) over one batch of the
Mamba-1.4B-shaped layer workload (batch 4, D 4096, N 16, L 4096, bf16
inputs, fp32 state and output) with inputs resident in HBM.  W untimed steps,
then exactly K steps bracketed by a barrier and a device synchronise on both
sides, timed with CUDA events on the launching stream; the time is the max
over ranks.  The working set (672 MB of inputs and outputs) is larger than
the 126 MB L2, so no step finds the previous step's data in L2.

The line also carries ``per_config``: every named workload (tiny fp32,
130M-shaped layer, 1.4B-shaped layer, long-context, audio-length) timed the
same way for a short run, with its HBM and exponential-unit fractions and
its error against the fp64 oracle on a sample of channels.  The default
workload's own error is measured on every output element.

Under torchrun (N > 1) every rank runs an independent replica of the
workload on its own GPU (the scan needs no exchange between GPUs) and
``value`` is the bytes moved by all ranks divided by the slowest rank's time.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
instead (the only other place the bench runs it), on a bounded sample of the
same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import faulthandler
import hashlib
import glob
import json
import math
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

import workloads  # noqa: E402

METRIC = ("selective-scan HBM GB/s (fraction of B200 peak); "
          "B·D·L·N state-updates/s")
DEFAULT_WORKLOAD = "mamba1.4b-layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "roofline_traffic.json")

REASON_BITS = [
    (0x1, "gpu_idle"), (0x2, "applications_clocks_setting"),
    (0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x10, "sync_boost"),
    (0x20, "sw_thermal_slowdown"), (0x40, "hw_thermal_slowdown"),
    (0x80, "hw_power_brake_slowdown"), (0x100, "display_clock_setting"),
]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=[w.name for w in workloads.WORKLOADS])
    ap.add_argument("--out-dtype", choices=["f32", "bf16"], default="f32",
                    help="dtype of y (f32 is the metric's configuration)")
    ap.add_argument("--varlen", type=int, default=0,
                    help="pack this many independent sequences into every row "
                         "(seeded random offsets; 0 = one sequence per row)")
    ap.add_argument("--checkpoints", action="store_true",
                    help="forward: also write the backward's state checkpoints; "
                         "bwd: start from checkpoints written by a forward scan")
    ap.add_argument("--trapezoid", action="store_true",
                    help="three-term trapezoidal update instead of the Euler one")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd", "decode", "ssd"],
                    default="fwd",
                    help="bwd times the backward scan (gradients of all inputs); "
                         "decode times one-token state updates; ssd times the "
                         "Mamba-2 chunked scan on the tensor cores")
    ap.add_argument("--ssd-workload", default="mamba2-2.7b-layer",
                    choices=[w.name for w in workloads.SSD_WORKLOADS])
    ap.add_argument("--decode-batch", type=int, default=1024,
                    help="batch rows of one decode step (the workload's dim and dstate)")
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the short runs of the other named workloads")
    ap.add_argument("--parity", choices=["all", "sample", "none"], default="all",
                    help="error of the timed output against the fp64 oracle: every "
                         "element (all), 64 channels (sample) or not at all")
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="CPU time budget of --impl reference (default: "
                         "3 s per step, between 20 and 120 s)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- helpers


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak for a kernel timed in a loop of launches: the
    sustained cuBLAS figure of the measured peaks, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        return 1400.0, "fallback (sustained)"


# the sources each timed kernel is compiled from
KERNEL_SOURCES = {
    "fwd": ("device_math.cuh", "scan_fwd.cu", "scan_fwd.cuh"),
    "bwd": ("device_math.cuh", "scan_bwd.cu", "scan_bwd.cuh"),
    "decode": ("device_math.cuh", "state_update.cu"),
    "ssd": ("device_math.cuh", "ssd_fwd.cu"),
}


def kernel_source_hash(kernel: str = "fwd") -> str:
    """Hash of the source files one kernel is built from (a profile's
    counters stay valid while it is unchanged)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_48_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "fwd"):
    """DRAM bytes per launch from the committed ncu summary, or None when
    the kernel changed since the counters were taken.  Entries are keyed by
    workload name, prefixed with the kernel for the passes other than the
    forward scan and the SSD scan ("bwd:mamba130m-layer")."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        e = d.get(workload) if kernel in ("fwd", "ssd") else d.get(f"{kernel}:{workload}")
        if e and e.get("kernel_source_hash") == kernel_source_hash(kernel):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def varlen_offsets(L: int, n: int) -> list:
    """n sequences packed into a row of L steps: seeded random interior
    offsets, the same for every row."""
    rng = np.random.default_rng(48000 + n)
    cuts = rng.choice(np.arange(1, L), size=min(n - 1, L - 1), replace=False)
    return [0] + sorted(int(c) for c in cuts) + [L]


def sfu_ops_per_step(w) -> int:
    """Special-function operations one forward scan needs: the decay
    exp(Delta A) of every state update, the exponential of softplus and the
    exponential and reciprocal of silu(z) per (b, d, t)."""
    per_elem = (1 if w.softplus else 0) + (2 if w.has_z else 0)
    return w.state_updates + per_elem * w.batch * w.dim * w.seqlen


def out_bytes(out_dtype: str) -> int:
    return 2 if out_dtype == "bf16" else 4


def workload_config(w, out_dtype="f32") -> dict:
    nbytes = w.algorithmic_bytes(out_bytes(out_dtype))
    return {"workload": w.name, "batch": w.batch, "dim": w.dim,
            "dstate": w.dstate, "seqlen": w.seqlen, "in_dtype": w.in_dtype,
            "out_dtype": out_dtype, "gate": "silu(z)" if w.has_z else "none",
            "l2": (f"inputs+outputs {nbytes / 1e6:.0f} MB per "
                   "step, larger than the 126 MB L2; no flush")}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, cuda_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            handle = None
            uuid = getattr(torch.cuda.get_device_properties(cuda_index), "uuid", None)
            if isinstance(uuid, str) and uuid:
                # NVML wants the "GPU-" prefixed form; only a str is passed on
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(
                        uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
                except Exception:
                    handle = None
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(int(cuda_index))
            self._handle = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self._handle, n.NVML_CLOCK_SM)
                reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": [name for bit, name in REASON_BITS if bits & bit],
                "samples": len(self.samples)}


def reduce_max(value: float, world: int) -> float:
    """Max over ranks (all ranks call this in the same order)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def whole_job_gbs(bytes_per_step: int, steps: int, world: int,
                  max_ms: float) -> float:
    return bytes_per_step * steps * world / (max_ms * 1e-3) / 1e9


# ------------------------------------------------------- oracle (CPU) legs


def _oracle_sample_inputs(inp: dict, channels: int, w):
    """First `channels` channels in (b, d) order, as float64 host arrays,
    grouped per batch row (contiguous d ranges)."""
    groups = []
    left = channels
    b = 0
    while left > 0 and b < w.batch:
        nd = min(left, w.dim)
        sl = lambda t: None if t is None else t[b:b + 1, :nd].detach().cpu().double().numpy()
        pd = lambda t: None if t is None else t[:nd].detach().cpu().double().numpy()
        groups.append(dict(u=sl(inp["u"]), delta=sl(inp["delta"]), z=sl(inp["z"]),
                           B=inp["B"][b:b + 1].detach().cpu().double().numpy(),
                           C=inp["C"][b:b + 1].detach().cpu().double().numpy(),
                           A=inp["A"][:nd].detach().cpu().double().numpy(),
                           D=pd(inp["D"]), delta_bias=pd(inp["delta_bias"])))
        left -= nd
        b += 1
    return groups


def _run_oracle_groups(groups, w, **kw):
    import oracle
    return [oracle.selective_scan(g["u"], g["delta"], g["A"], g["B"], g["C"],
                                  D=g["D"], z=g["z"], delta_bias=g["delta_bias"],
                                  delta_softplus=w.softplus, **kw)
            for g in groups]


def _calibrate_oracle(inp, w) -> float:
    """Seconds of wall time per channel with all oracle threads busy."""
    import oracle
    threads = oracle.num_threads()
    probe = max(1, min(threads, w.batch * w.dim))
    groups = _oracle_sample_inputs(inp, probe, w)
    t0 = time.perf_counter()
    _run_oracle_groups(groups, w)
    dt = time.perf_counter() - t0
    return dt / probe


def oracle_timing(inp, w, seconds: float, steps: int = 1, warmup: int = 0):
    """Time the oracle on a bounded sample; returns (GB/s, updates/s,
    channels per step, threads, total seconds)."""
    import oracle
    threads = oracle.num_threads()
    per_ch = _calibrate_oracle(inp, w)
    per_step = seconds / max(1, steps + warmup)
    ch = int(max(1, min(w.batch * w.dim, round(per_step / per_ch))))
    groups = _oracle_sample_inputs(inp, ch, w)
    for _ in range(warmup):
        _run_oracle_groups(groups, w)
    t0 = time.perf_counter()
    for _ in range(steps):
        _run_oracle_groups(groups, w)
    total = time.perf_counter() - t0
    share = ch / (w.batch * w.dim)
    gbs = w.algorithmic_bytes() * share * steps / total / 1e9
    ups = w.state_updates * share * steps / total
    return gbs, ups, ch, threads, total


def sample_max_norm_err(y, inp, w, channels: int, **oracle_kw) -> float:
    """max |y - y_oracle| / max |y_oracle| over the first `channels`
    channels of the batch (fp64 oracle on the same inputs; ``oracle_kw``
    passes cu_seqlens / trapezoid on)."""
    groups = _oracle_sample_inputs(inp, channels, w)
    worst, scale = 0.0, 0.0
    for b, (g, ref) in enumerate(zip(groups, _run_oracle_groups(groups, w, **oracle_kw))):
        got = y[b:b + 1, :ref.shape[1]].detach().float().cpu().double().numpy()
        worst = max(worst, float(np.abs(got - ref).max()))
        scale = max(scale, float(np.abs(ref).max()))
    return worst / scale if scale > 0 else worst


def all_elements_error(y, inp, w, block: int = 512) -> dict:
    """Error statistics of y against the oracle on every element (the
    oracle run a block of channels of one batch row at a time)."""
    import oracle
    from oracle.compare import ErrorStats
    st = ErrorStats()
    f = lambda t, b, d0, d1: None if t is None else \
        t[b:b + 1, d0:d1].detach().float().cpu().double().numpy()
    c = lambda t, d0, d1: None if t is None else t[d0:d1].detach().float().cpu().double().numpy()
    for b in range(w.batch):
        Bh = inp["B"][b:b + 1].detach().float().cpu().double().numpy()
        Ch = inp["C"][b:b + 1].detach().float().cpu().double().numpy()
        for d0 in range(0, w.dim, block):
            d1 = min(w.dim, d0 + block)
            ref = oracle.selective_scan(f(inp["u"], b, d0, d1), f(inp["delta"], b, d0, d1),
                                        c(inp["A"], d0, d1), Bh, Ch, D=c(inp["D"], d0, d1),
                                        z=f(inp["z"], b, d0, d1),
                                        delta_bias=c(inp["delta_bias"], d0, d1),
                                        delta_softplus=w.softplus)
            st.add(f(y, b, d0, d1), ref)
    return st.summary()


def single_thread_oracle(seconds: float = 4.0) -> dict:
    """The oracle on one core: the whole tiny fp32 workload, and a bounded
    sample of whole channels of the 130M-shaped layer; GB/s as the sample's
    share of the workload's algorithmic bytes per second."""
    import oracle
    out = {}
    threads = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        for name in ("tiny-fp32", "mamba130m-layer"):
            w = workloads.BY_NAME[name]
            inp = workloads.make_inputs(w, device="cpu")
            per_ch = _calibrate_oracle(inp, w)
            ch = int(max(1, min(w.batch * w.dim, round(seconds / 2 / per_ch))))
            groups = _oracle_sample_inputs(inp, ch, w)
            t0 = time.perf_counter()
            _run_oracle_groups(groups, w)
            secs = time.perf_counter() - t0
            share = ch / (w.batch * w.dim)
            out[name] = {"value": w.algorithmic_bytes() * share / secs / 1e9, "unit": "GB/s",
                         "state_updates_per_s": w.state_updates * share / secs,
                         "cores": 1, "sample": f"{ch} of {w.batch * w.dim} channels, "
                                               f"full length L={w.seqlen}, {secs:.2f} s"}
    finally:
        oracle.set_num_threads(threads)
    return out


def ssd_sample_max_norm_err(y, inp, w) -> float:
    """The same for the SSD scan: the heads of batch row 0's first group."""
    import oracle
    g = _ssd_sample(inp, w, w.nheads // w.ngroups)[0]
    ref = oracle.ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                          dt_bias=g["dt_bias"], dt_softplus=w.softplus)
    got = y[0:1, :, :ref.shape[2]].detach().float().cpu().double().numpy()
    scale = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    return err / scale if scale > 0 else err


def _ssd_sample(inp: dict, w, heads: int) -> list:
    """The first `heads` (batch row, head) pairs in (b, h) order at full
    length, as float64 host arrays grouped per batch row.  Counts are
    whole groups of heads, so each slice keeps its heads' group of B, C."""
    hpg = w.nheads // w.ngroups
    heads = max(hpg, (heads // hpg) * hpg)
    out, left, b = [], heads, 0
    while left > 0 and b < w.batch:
        k = min(left, w.nheads)
        f = lambda t: t.detach().cpu().double().numpy()
        hsel = lambda t: None if t is None else f(t[:k])
        out.append(dict(x=f(inp["x"][b:b + 1, :, :k]), dt=f(inp["dt"][b:b + 1, :, :k]),
                        A=hsel(inp["A"]), D=hsel(inp["D"]), dt_bias=hsel(inp["dt_bias"]),
                        z=None if inp["z"] is None else f(inp["z"][b:b + 1, :, :k]),
                        B=f(inp["B"][b:b + 1, :, :k // hpg]),
                        C=f(inp["C"][b:b + 1, :, :k // hpg])))
        left -= k
        b += 1
    return out


def _run_ssd_oracle(groups, w):
    import oracle
    for g in groups:
        oracle.ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                        dt_bias=g["dt_bias"], dt_softplus=w.softplus)


def ssd_oracle_timing(inp, w, seconds: float, out_b: int = 4, steps: int = 1,
                      warmup: int = 0):
    """Time the SSD oracle on a bounded sample of whole (batch row, head)
    sequences, `seconds` spread over warmup + steps passes; returns (GB/s,
    heads sampled per step, threads, seconds of the timed steps)."""
    import oracle
    threads = oracle.num_threads()
    hpg = w.nheads // w.ngroups
    probe = max(hpg, (max(1, threads) // hpg) * hpg)
    t0 = time.perf_counter()
    _run_ssd_oracle(_ssd_sample(inp, w, probe), w)
    per_head = (time.perf_counter() - t0) / probe
    per_step = seconds / max(1, steps + warmup)
    heads = int(max(1, min(w.batch * w.nheads, round(per_step / max(per_head, 1e-9)))))
    groups = _ssd_sample(inp, w, heads)
    heads = sum(g["x"].shape[2] for g in groups)
    for _ in range(warmup):
        _run_ssd_oracle(groups, w)
    t0 = time.perf_counter()
    for _ in range(steps):
        _run_ssd_oracle(groups, w)
    total = time.perf_counter() - t0
    share = heads / (w.batch * w.nheads)
    return w.algorithmic_bytes(out_b) * share * steps / total / 1e9, heads, threads, total


# ------------------------------------------------------------- our arm


def bwd_algorithmic_bytes(w) -> int:
    """Every input of the backward pass read once (u, delta, z, B, C in the
    input dtype, dy fp32) and every gradient written once in fp32."""
    si = 2 if w.in_dtype == "bf16" else 4
    bdl = w.batch * w.dim * w.seqlen
    per_ch = 2 * si + (si + 4 if w.has_z else 0) + 4 + 2 * 4
    bnl = w.batch * w.dstate * w.seqlen
    return bdl * per_ch + bnl * 2 * (si + 4) + w.dim * w.dstate * 8


def run_bwd(args, rank, world, local_rank):
    import selective_state_space_48_b200 as sss
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.BY_NAME[args.workload]
    inp = workloads.make_inputs(w, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(48000)
    dy = torch.randn(w.batch, w.dim, w.seqlen, generator=g, device=dev)

    ck = None
    cu = (torch.tensor(varlen_offsets(w.seqlen, args.varlen), dtype=torch.int32, device=dev)
          if args.varlen else None)
    if args.checkpoints and cu is not None:
        raise SystemExit("--checkpoints and --varlen do not combine for the backward")
    if args.checkpoints:
        ck = sss.scan_checkpoints(w.batch, w.dim, w.dstate, w.seqlen, dev)
        sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=w.softplus, checkpoints=ck)

    def step():
        sss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=w.softplus, workspace=ws, checkpoints=ck,
                               cu_seqlens=cu)

    # workspace sized once (the size depends on the shapes only)
    nb = ctypes.c_size_t(0)
    a = sss.ScanBwdArgs()
    a.batch, a.dim, a.dstate, a.seqlen = w.batch, w.dim, w.dstate, w.seqlen
    a.in_dtype = sss.MSS_BF16 if w.in_dtype == "bf16" else sss.MSS_F32
    for f in ("u", "delta", "A", "B", "C", "dy", "du", "ddelta", "dA", "dB", "dC"):
        setattr(a, f, 256)  # only checked for presence and alignment here
    if sss.load_library().mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(nb)):
        raise RuntimeError("mss_scan_bwd_workspace_size failed")
    ws = torch.empty(int(nb.value), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    stream = torch.cuda.current_stream(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(world)
    max_ms = reduce_max(t0.elapsed_time(t1), world)
    nbytes = bwd_algorithmic_bytes(w)
    value = whole_job_gbs(nbytes, K, world, max_ms)
    peak, src = measured_peaks()
    line = {
        "metric": "selective-scan backward HBM GB/s; B*D*L*N state updates/s",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(w), **{"pass": "bwd"},
                       **({"from_checkpoints": True} if args.checkpoints else {}),
                       **({"sequences_per_row": args.varlen} if args.varlen else {})),
        "state_updates_per_s": w.state_updates * K * world / (max_ms * 1e-3),
        "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak,
                     "unit": "GB/s", "frac": value / world / peak,
                     "peak_source": src,
                     "traffic": (None if (args.checkpoints or args.varlen)
                                 else profiled_traffic(w.name, "bwd")),
                     "algorithmic_bytes_per_launch": nbytes},
        "e2e": None, "gpu_launches": K, "clocks": clocks.summary(),
        "kernel_source_hash": kernel_source_hash("bwd"),
    }
    if rank == 0:
        try:
            line["max_norm_err"] = bwd_row_max_norm_err(sss, inp, dy, w, ws, ck, cu)
            line["max_norm_err_sample"] = ("batch row 0: du, ddelta, dz, dB, dC vs the fp64 "
                                           "oracle backward (max over the five)")
        except Exception as ex:  # reported, never fatal to the timing line
            print(f"parity sample failed: {ex}", file=sys.stderr)
        print(json.dumps(line), flush=True)


def bwd_row_max_norm_err(sss, inp, dy, w, ws, ck, cu=None) -> float:
    """The backward's per-row gradients of batch row 0 against the oracle
    backward of that row alone (dA, dD, ddelta_bias sum over all rows and
    are left to the tests)."""
    import oracle
    g = sss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=w.softplus, workspace=ws, checkpoints=ck,
                               cu_seqlens=cu)
    torch.cuda.synchronize()
    row = lambda t: None if t is None else t[:1].detach().float().cpu().double().numpy()
    par = lambda t: None if t is None else t.detach().float().cpu().double().numpy()
    ref = oracle.selective_scan_bwd(row(inp["u"]), row(inp["delta"]), par(inp["A"]),
                                    row(inp["B"]), row(inp["C"]), row(dy), D=par(inp["D"]),
                                    z=row(inp["z"]), delta_bias=par(inp["delta_bias"]),
                                    delta_softplus=w.softplus,
                                    cu_seqlens=None if cu is None else cu.cpu().tolist())
    worst = 0.0
    for k in ("du", "ddelta", "dz", "dB", "dC"):
        if ref[k] is None:
            continue
        got = g[k][:1].cpu().double().numpy()
        worst = max(worst, float(np.abs(got - ref[k]).max() / np.abs(ref[k]).max()))
    return worst


def decode_algorithmic_bytes(batch, dim, dstate, in_bytes) -> int:
    """One decode step: the fp32 state read and written once, x, dt, z in
    and y (fp32) out per channel, B and C per batch row, A, D, dt_bias."""
    return (batch * dim * (8 * dstate + 3 * in_bytes + 4) + batch * dstate * 2 * in_bytes
            + dim * dstate * 4 + dim * 8)


def run_decode(args, rank, world, local_rank):
    import selective_state_space_48_b200 as sss
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.BY_NAME[args.workload]
    bt, D, N = args.decode_batch, w.dim, w.dstate
    dt_ = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    g = torch.Generator(device=dev)
    g.manual_seed(48000)
    rnd = lambda *shape: torch.randn(*shape, generator=g, device=dev)
    state = rnd(bt, D, N)
    x, dtv, z = rnd(bt, D).to(dt_), rnd(bt, D).to(dt_), rnd(bt, D).to(dt_)
    B, C = rnd(bt, N).to(dt_), rnd(bt, N).to(dt_)
    A = -torch.arange(1, N + 1, device=dev, dtype=torch.float32).repeat(D, 1)
    Dv = rnd(D)
    bias = torch.log(torch.expm1(torch.rand(D, generator=g, device=dev) * 0.099 + 1e-3))
    y = torch.empty(bt, D, device=dev)

    def step():
        sss.selective_state_update(state, x, dtv, A, B, C, D=Dv, z=z, dt_bias=bias, y=y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    stream = torch.cuda.current_stream(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(world)
    max_ms = reduce_max(t0.elapsed_time(t1), world)
    nbytes = decode_algorithmic_bytes(bt, D, N, 2 if dt_ == torch.bfloat16 else 4)
    value = whole_job_gbs(nbytes, K, world, max_ms)
    peak, src = measured_peaks()
    line = {
        "metric": "selective state update (decode) HBM GB/s; tokens/s",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "pass": "decode", "batch": bt, "dim": D,
                   "dstate": N, "in_dtype": w.in_dtype,
                   "l2": f"{nbytes / 1e6:.0f} MB per step"},
        "tokens_per_s": bt * K * world / (max_ms * 1e-3),
        "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak,
                     "unit": "GB/s", "frac": value / world / peak,
                     "peak_source": src,
                     "traffic": (profiled_traffic(f"{w.name}-{bt}rows", "decode")
                                 if bt == 1024 else None),
                     "algorithmic_bytes_per_launch": nbytes},
        "e2e": None, "gpu_launches": K, "clocks": clocks.summary(),
        "kernel_source_hash": kernel_source_hash("decode"),
    }
    if rank == 0:
        try:
            import oracle
            h = lambda t: t.detach().float().cpu().double().numpy()
            st0 = state.clone()
            s_ref, y_ref = oracle.selective_state_update(
                h(st0), h(x), h(dtv), h(A), h(B), h(C), D=h(Dv), z=h(z), dt_bias=h(bias))
            yv = sss.selective_state_update(st0, x, dtv, A, B, C, D=Dv, z=z, dt_bias=bias)
            torch.cuda.synchronize()
            line["max_norm_err"] = max(
                float(np.abs(h(yv) - y_ref).max() / np.abs(y_ref).max()),
                float(np.abs(h(st0) - s_ref).max() / np.abs(s_ref).max()))
            line["max_norm_err_sample"] = "one more step, every y and state element"
        except Exception as ex:  # reported, never fatal to the timing line
            print(f"parity sample failed: {ex}", file=sys.stderr)
        print(json.dumps(line), flush=True)


# measured on this machine's B200s with the library's own probes: results per
# clock per SM of ex2.approx alone, and of the best mix of ex2.approx with
# the FMA-pipe polynomial exp2 (three on the special-function unit to one
# polynomial)
SFU_PER_CLK_SM = 16.0
EXP_MIX_PER_CLK_SM = 20.5
L2_BYTES = 126 * 1024 * 1024


def exp_unit_bound(w, kernel_ms: float, sm_mhz: float) -> dict:
    """The special-function-unit roofline of one scan: one ex2 per state
    update plus the softplus ex2 and the silu ex2 and reciprocal per
    (b, d, t), against 16 per clock per SM; and the exponentials alone
    against the measured rate of the best special-function / FMA-pipe mix
    (the ceiling if part of the decays moved to the polynomial)."""
    ops = sfu_ops_per_step(w)
    clk = sm_mhz * 1e6
    sfu_peak = SFU_PER_CLK_SM * 148 * clk / 1e12
    mix_peak = EXP_MIX_PER_CLK_SM * 148 * clk / 1e12
    achieved = ops / (kernel_ms * 1e-3) / 1e12
    exps = w.state_updates / (kernel_ms * 1e-3) / 1e12
    return {"achieved": achieved, "peak": sfu_peak, "unit": "Tops/s",
            "frac": achieved / sfu_peak, "algorithmic_ops_per_launch": ops,
            "peak_source": ("derived: 16 special-function results per clock per SM "
                            "(measured) x 148 SMs x the sampled SM clock"),
            "decay_exps_per_s": exps * 1e12,
            "frac_of_exp_mix": exps / mix_peak,
            "exp_mix_peak": mix_peak,
            "exp_mix_source": ("derived: 20.5 exponentials per clock per SM measured for "
                               "3 ex2.approx : 1 FMA-pipe polynomial, x 148 SMs x clock")}


def _scan_setup(sss, w, inp, dev, out_dtype="f32", varlen=0, trapezoid=False,
                checkpoints=False):
    ydt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    y = torch.empty((w.batch, w.dim, w.seqlen), dtype=ydt, device=dev)
    ck = sss.scan_checkpoints(w.batch, w.dim, w.dstate, w.seqlen, dev) if checkpoints else None
    cu_t = None
    if varlen > 0:
        cu_t = torch.tensor(varlen_offsets(w.seqlen, varlen), dtype=torch.int32, device=dev)
    sargs = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=w.softplus, y=y, cu_seqlens=cu_t,
                               trapezoid=trapezoid, checkpoints=ck)
    ws_bytes = sss.scan_workspace_size(sargs)
    ws = sss.alloc_workspace(ws_bytes, dev)
    if ws is not None:
        sargs.workspace = ws.data_ptr()
        sargs.workspace_bytes = ws_bytes
    return dict(y=y, ck=ck, cu=cu_t, args=sargs, ws=ws)


def _timed(step, stream, steps, flush=None):
    """Per-step CUDA events around `steps` calls (an L2 flush between them,
    outside the events, when given); returns (total ms from the first to
    the last event, mean ms per step inside the events)."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for a, b in ev:
        if flush is not None:
            flush.add_(1)
        a.record(stream)
        step()
        b.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    return t_start.elapsed_time(t_end), sum(a.elapsed_time(b) for a, b in ev) / steps


def per_config(args, dev, sss, rank, sm_mhz) -> dict:
    """Every named workload timed for a short run (inputs resident; an L2
    flush between steps for workloads that fit in L2), with its HBM and
    exponential-unit fractions and its error against the oracle on the
    first 64 channels."""
    lib = sss.load_library()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    peak, _ = measured_peaks()
    out = {}
    flush = None
    for w in workloads.WORKLOADS:
        inp = workloads.make_inputs(w, device=dev)
        st = _scan_setup(sss, w, inp, dev)
        argp = ctypes.byref(st["args"])
        nbytes = w.algorithmic_bytes()
        small = nbytes < 2 * L2_BYTES
        if small and flush is None:
            flush = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)

        def step():
            rc = lib.mamba_selective_scan_fwd(argp, sh)
            if rc != 0:
                raise sss.MssError(rc, "mamba_selective_scan_fwd")

        _, warm_ms = _timed(step, stream, 3, flush if small else None)
        steps = int(min(300, max(10, round(150.0 / max(warm_ms, 1e-3)))))
        _, kms = _timed(step, stream, steps, flush if small else None)
        if lib.mss_scan_status(argp, sh) != 0:
            raise RuntimeError(f"device-side status error ({w.name})")
        entry = {"ms_per_step": kms, "steps": steps,
                 "value": nbytes / (kms * 1e-3) / 1e9, "unit": "GB/s",
                 "hbm_frac": nbytes / (kms * 1e-3) / 1e9 / peak,
                 "state_updates_per_s": w.state_updates / (kms * 1e-3),
                 "exp_unit_frac": exp_unit_bound(w, kms, sm_mhz)["frac"],
                 "l2": ("flushed between steps (256 MB write)" if small
                        else "inputs+outputs larger than L2, no flush"),
                 "sequence_split": sss.scan_workspace_size(st["args"]) > 0}
        # a split scan is three kernels (chunks, prefix over the chunks, carry)
        entry["launches_per_step"] = 3 if entry["sequence_split"] else 1
        if rank == 0:
            try:
                entry["max_norm_err"] = sample_max_norm_err(st["y"], inp, w, 64)
                entry["max_norm_err_sample"] = "first 64 channels, full length"
            except Exception as ex:  # reported, never fatal to the timing
                print(f"parity sample failed ({w.name}): {ex}", file=sys.stderr)
        out[w.name] = entry
        del inp, st
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import selective_state_space_48_b200 as sss
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.BY_NAME[args.workload]
    inp = workloads.make_inputs(w, device=dev)
    st = _scan_setup(sss, w, inp, dev, args.out_dtype, args.varlen, args.trapezoid,
                     args.checkpoints)
    y, ck, cu_t, ws, sargs = st["y"], st["ck"], st["cu"], st["ws"], st["args"]
    lib = sss.load_library()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    argp = ctypes.byref(sargs)

    def step():
        rc = lib.mamba_selective_scan_fwd(argp, sh)
        if rc != 0:
            raise sss.MssError(rc, "mamba_selective_scan_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if lib.mss_scan_status(argp, sh) != 0:
        raise RuntimeError("device-side status error during warm-up")

    K = args.steps
    clocks = ClockSampler(local_rank)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    local_ms, kernel_ms = _timed(step, stream, K)
    clocks.stop()
    barrier(world)
    max_ms = reduce_max(local_ms, world)
    max_kernel_ms = reduce_max(kernel_ms, world)
    if lib.mss_scan_status(argp, sh) != 0:
        raise RuntimeError("device-side status error in the timed region")

    bytes_step = w.algorithmic_bytes(out_bytes(args.out_dtype))
    value = whole_job_gbs(bytes_step, K, world, max_ms)
    # a split scan is three kernels per step (chunks, prefix over the chunks,
    # carry); the roofline then covers the three together
    launches_per_step = 3 if sss.scan_workspace_size(sargs) > 0 else 1
    updates = w.state_updates * K * world / (max_ms * 1e-3)

    # ---- end to end through the public API with host buffers.  Every step
    # uploads its inputs from pinned host memory, scans and reads y back;
    # two sets of device buffers and three streams let step i+1's upload and
    # step i-1's read-back run while step i is scanned (the copy engines of
    # both directions and the SMs work at once).  A step's inputs sit in one
    # pinned host slab (each at a 256-byte offset) and go up as one copy into
    # a device slab whose views the scan reads.
    names = ["u", "delta", "z", "B", "C", "A", "D", "delta_bias"]
    src = {k: inp[k].detach() for k in names if inp[k] is not None}
    nbytes_of = {k: t.numel() * t.element_size() for k, t in src.items()}
    offs, slab_bytes = {}, 0
    for k in src:
        offs[k] = slab_bytes
        slab_bytes += (nbytes_of[k] + 255) // 256 * 256
    host_slab = torch.empty(slab_bytes, dtype=torch.uint8).pin_memory()
    for k, t in src.items():
        host_slab[offs[k]:offs[k] + nbytes_of[k]].copy_(
            t.contiguous().view(-1).view(torch.uint8).cpu())
    dev_slabs = [torch.empty(slab_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]

    def slab_views(slab):
        v = {k: slab[offs[k]:offs[k] + nbytes_of[k]].view(t.dtype).view(t.shape)
             for k, t in src.items()}
        return {k: v.get(k) for k in inp}

    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    h2d = slab_bytes
    d2h = y.numel() * y.element_size()
    sets = [slab_views(dev_slabs[0]), slab_views(dev_slabs[1])]
    ys = [y, torch.empty_like(y)]
    s_up, s_cmp, s_dn = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    up_done, cmp_done, dn_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    Ke = max(1, args.e2e_steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for st in (s_up, s_cmp, s_dn):
        st.wait_stream(stream)
    for i in range(Ke):
        j = i % 2
        d = sets[j]
        if i >= 2:
            s_up.wait_event(cmp_done[j])  # set j's scan of step i-2 is done
        with torch.cuda.stream(s_up):
            dev_slabs[j].copy_(host_slab, non_blocking=True)
        up_done[j].record(s_up)
        s_cmp.wait_event(up_done[j])
        if i >= 2:
            s_cmp.wait_event(dn_done[j])  # y set j was read back
        sss.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"],
                               z=d["z"], delta_bias=d["delta_bias"],
                               delta_softplus=w.softplus, y=ys[j], workspace=ws,
                               cu_seqlens=cu_t, trapezoid=args.trapezoid,
                               checkpoints=ck, stream=s_cmp)
        cmp_done[j].record(s_cmp)
        s_dn.wait_event(cmp_done[j])
        with torch.cuda.stream(s_dn):
            y_host[j].copy_(ys[j], non_blocking=True)
        dn_done[j].record(s_dn)
    stream.wait_stream(s_dn)
    stream.wait_stream(s_up)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = reduce_max(e0.elapsed_time(e1), world)
    e2e_value = whole_job_gbs(bytes_step, Ke, world, e2e_ms)
    # the link's own bound for the same bytes: the step's uploads and its
    # read-back as plain copies, both directions at once, no scan
    def copies_only():
        s_up.wait_stream(stream)
        s_dn.wait_stream(stream)
        with torch.cuda.stream(s_up):
            dev_slabs[1].copy_(host_slab, non_blocking=True)
        with torch.cuda.stream(s_dn):
            y_host[1].copy_(ys[1], non_blocking=True)
        stream.wait_stream(s_up)
        stream.wait_stream(s_dn)
    copies_only()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(3):
        copies_only()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    link_ms = reduce_max(e0.elapsed_time(e1), world) / 3
    link_value = whole_job_gbs(bytes_step, 1, world, link_ms)
    del sets, dev_slabs, ys[1]

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, ups, ch, threads, total = oracle_timing(inp, w, args.cpu_seconds)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "state_updates_per_s": ups,
               "sample": (f"{ch} of {w.batch * w.dim} channels, full length "
                          f"L={w.seqlen}, one pass, {total:.1f} s wall, "
                          "fp64 C oracle with OpenMP over channels; GB/s = the "
                          "sample's share of the step's algorithmic bytes / time"),
               "single_thread": single_thread_oracle()}

    # ---- parity of the timed output against the fp64 oracle
    err, parity = None, None
    okw = {}
    if args.varlen:
        okw["cu_seqlens"] = varlen_offsets(w.seqlen, args.varlen)
    if args.trapezoid:
        okw["trapezoid"] = True
    if rank == 0 and args.parity != "none":
        try:
            if args.parity == "all" and not okw:
                parity = all_elements_error(y, inp, w)
                parity["sample"] = "every output element, vs the fp64 oracle"
                err = parity["max_norm_err"]
            else:
                err = sample_max_norm_err(y, inp, w, 64, **okw)
                parity = {"max_norm_err": err,
                          "sample": "first 64 channels, full length, vs the fp64 oracle"}
        except Exception as ex:  # reported, never fatal to the timing line
            print(f"parity check failed: {ex}", file=sys.stderr)
    del inp, st, host_slab, y_host
    torch.cuda.empty_cache()

    peak, peak_kind = measured_peaks()
    achieved = bytes_step / (max_kernel_ms * 1e-3) / 1e9
    clk = clocks.summary()
    sm_mhz = clk.get("sm_mhz") or 1965.0
    pcfg = None
    # per-workload lines on one GPU only (each rank would time the same
    # replicas again under torchrun)
    if world == 1 and not args.no_per_config and not (args.varlen or args.trapezoid
                                                      or args.checkpoints):
        pcfg = per_config(args, dev, sss, rank, sm_mhz)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": max_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": dict(workload_config(w, args.out_dtype),
                       **({"sequences_per_row": args.varlen} if args.varlen else {}),
                       **({"update": "trapezoidal"} if args.trapezoid else {}),
                       **({"writes_checkpoints": True} if args.checkpoints else {})),
        "state_updates_per_s": updates,
        "max_norm_err": err,
        "parity": parity,
        "frac_of_nominal_8tbs": value / world / NOMINAL_HBM_GBS,
        "frac_of_measured_hbm": value / world / peak,
        # the metric's roofline: algorithmic HBM bytes per launch over the
        # kernel's own time (per-step events on the launching stream)
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "traffic": (profiled_traffic(w.name)
                                 if not (args.varlen or args.trapezoid or args.checkpoints
                                         or args.out_dtype != "f32") else None),
                     "algorithmic_bytes_per_launch": bytes_step,
                     "kernel_ms": max_kernel_ms,
                     **({"covers": "the step's three launches (chunks, prefix, carry)"}
                        if launches_per_step > 1 else {})},
        # the bound that binds this scan: the special-function unit (one
        # ex2 per state update)
        "exp_unit": exp_unit_bound(w, max_kernel_ms, sm_mhz),
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke,
                "overlap": "upload of step i+1 and read-back of step i-1 during the scan of step i",
                "link_bound": {"value": link_value, "unit": "GB/s",
                               "what": "the same uploads and read-back as plain pinned copies, "
                                       "both directions at once, no scan"}},
        "gpu_launches": K * launches_per_step,
        "launches_per_step": launches_per_step,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
        "kernel_source_hash": kernel_source_hash("fwd"),
    }
    if pcfg is not None:
        line["per_config"] = pcfg
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# -------------------------------------------------------- reference arm


SSD_METRIC = "Mamba-2 SSD chunked scan HBM GB/s; tokens/s"


def ssd_config(w, out_dtype: str) -> dict:
    return {"workload": w.name, "pass": "ssd", "batch": w.batch, "seq_len": w.seqlen,
            "nheads": w.nheads, "headdim": w.headdim, "ngroups": w.ngroups,
            "dstate": w.dstate, "chunk": 128, "y_dtype": out_dtype}


def run_reference_ssd(args):
    """The SSD oracle as it stands, on this host's cores, each step a
    bounded sample (whole head sequences) of the SSD workload."""
    w = workloads.SSD_BY_NAME[args.ssd_workload]
    inp = workloads.make_ssd_inputs(w, seed=48100)
    budget = args.ref_seconds
    if budget is None:
        budget = min(120.0, max(20.0, 3.0 * (args.steps + args.warmup)))
    gbs, heads, threads, total = ssd_oracle_timing(inp, w, budget, out_bytes(args.out_dtype),
                                                   steps=args.steps, warmup=args.warmup)
    sample = (f"{heads} of {w.batch * w.nheads} (batch row, head) sequences per step, full "
              f"length L={w.seqlen}; fp64 C oracle, OpenMP over (batch row, head)")
    return {
        "impl": "reference", "metric": SSD_METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": ssd_config(w, args.out_dtype),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_reference(args):
    """The fp64 oracle as it stands, on this host's cores, each step a
    bounded sample (a share of the channels, full length) of the workload."""
    if args.pass_ == "ssd":
        return run_reference_ssd(args)
    w = workloads.BY_NAME[args.workload]
    inp = workloads.make_inputs(w, device="cpu")
    budget = args.ref_seconds
    if budget is None:
        budget = min(120.0, max(20.0, 3.0 * (args.steps + args.warmup)))
    gbs, ups, ch, threads, total = oracle_timing(inp, w, budget, steps=args.steps,
                                                 warmup=args.warmup)
    sample = (f"{ch} of {w.batch * w.dim} channels per step, full length "
              f"L={w.seqlen}; fp64 C oracle, OpenMP over channels")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": gbs,
        "unit": "GB/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total * 1e3 / max(1, args.steps),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(w),
        "state_updates_per_s": ups,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_ssd(args, rank, world, local_rank):
    import selective_state_space_48_b200 as sss
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.SSD_BY_NAME[args.ssd_workload]
    inp = workloads.make_ssd_inputs(w, seed=48100, device=dev)
    ody = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    y = torch.empty(w.batch, w.seqlen, w.nheads, w.headdim, dtype=ody, device=dev)
    # workspace sized once: it lets the last wave's sequences be cut into
    # pieces spread over the schedule (the library's rule, restated here
    # only to report it)
    ws_bytes = sss.ssd_workspace_size(sss.make_ssd_args(inp["x"], inp["dt"], inp["A"],
                                                        inp["B"], inp["C"]))
    ws = sss.alloc_workspace(ws_bytes, dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    waves, ncut = divmod(w.batch * w.nheads, sms)
    nch = (w.seqlen + 127) // 128
    parts = (min(max(2, (sms + ncut // 2) // ncut), waves + 1, nch, 8)
             if ws_bytes and ncut else 0)
    ncut = ncut if parts else 0

    def step():
        sss.ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                    z=inp["z"], dt_bias=inp["dt_bias"], dt_softplus=w.softplus, y=y,
                    workspace=ws if ws is not None else False)

    for _ in range(args.warmup):
        step()
    if sss.load_library().mss_ssd_status(None) != sss.MSS_OK:
        raise RuntimeError("SSD kernel reported a timeout")
    torch.cuda.synchronize(dev)
    K = args.steps
    stream = torch.cuda.current_stream(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(world)
    max_ms = reduce_max(t0.elapsed_time(t1), world)
    if sss.load_library().mss_ssd_status(None) != sss.MSS_OK:
        raise RuntimeError("SSD kernel reported a timeout in the timed region")
    nbytes = w.algorithmic_bytes(out_bytes(args.out_dtype))
    flops = w.chunk_flops()
    value = whole_job_gbs(nbytes, K, world, max_ms)
    peak, src = measured_peaks()
    tflops = flops * K / (max_ms * 1e-3) / 1e12
    tpeak, tsrc = measured_tensor_peak()
    line = {
        "metric": SSD_METRIC,
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": dict(ssd_config(w, args.out_dtype),
                       l2=f"inputs larger than L2 ({nbytes / 1e6:.0f} MB per step)"),
        "tokens_per_s": w.batch * w.seqlen * K * world / (max_ms * 1e-3),
        "schedule": {"ctas": w.batch * w.nheads + max(parts - 1, 0) * ncut,
                     "sequences_cut": ncut, "pieces_per_cut_sequence": parts},
        "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak,
                     "unit": "GB/s", "frac": value / world / peak,
                     "peak_source": src,
                     "traffic": (profiled_traffic(w.name, "ssd")
                                 if args.out_dtype == "f32" else None),
                     "algorithmic_bytes_per_launch": nbytes,
                     "tensor": {"achieved": tflops / world, "peak": tpeak,
                                "unit": "TFLOP/s", "frac": tflops / world / tpeak,
                                "peak_source": tsrc,
                                "algorithmic_flops_per_launch": flops}},
        "e2e": None, "gpu_launches": K, "clocks": clocks.summary(),
        "kernel_source_hash": kernel_source_hash("ssd"),
    }
    if rank == 0:
        try:
            line["max_norm_err"] = ssd_sample_max_norm_err(y, inp, w)
            line["max_norm_err_sample"] = (f"batch row 0, heads 0-{w.nheads // w.ngroups - 1}, "
                                           "full length, vs the fp64 oracle")
        except Exception as ex:  # reported, never fatal to the timing line
            print(f"parity sample failed: {ex}", file=sys.stderr)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, heads, threads, secs = ssd_oracle_timing(inp, w, args.cpu_seconds / 2,
                                                      out_bytes(args.out_dtype))
        line["cpu_baseline"] = {
            "value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": (f"{heads} of {w.batch * w.nheads} (batch row, head) sequences at "
                       f"full length L={w.seqlen}, one pass, {secs:.1f} s wall, fp64 C "
                       "oracle with OpenMP over (batch row, head); GB/s = the sample's "
                       "share of the step's algorithmic bytes / time")}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    try:
        faulthandler.enable()
    except (AttributeError, ValueError, OSError):
        pass  # stderr without a file descriptor (e.g. captured by a test)
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.pass_ == "bwd":
            run_bwd(args, rank, world, local_rank)
        elif args.pass_ == "decode":
            run_decode(args, rank, world, local_rank)
        elif args.pass_ == "ssd":
            run_ssd(args, rank, world, local_rank)
        else:
            line = run_ours(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
