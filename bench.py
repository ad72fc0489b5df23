#!/usr/bin/env python3
"""Benchmark of the B200 H-BitLinear forward path (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A pass is the whole per-token path -- RMSNorm, optional FWHT, activation
quantisation, ternary GEMM/GEMV, fp32 epilogue -- over one batch of the workload
(weights are packed once, before timing, as a deployment would).  A step is B
such passes over B batches (the input rotations in turn), B chosen before timing
so that one step holds at least 5 ms of device work (`config.batches_per_step`):
even a short run of timed steps then spans tens of clock samples.  The default
workload is the largest configuration that fits one GPU: the M = 8192 point of the
4096-hidden M-sweep, int4 absmean + FWHT, X Student-t(3) with 1 % outlier channels
x50, against Wo [4096 x 4096] and Wdown [4096 x 16384]; one pass runs the two
forwards (1.37 Tera integer ops).  The same line carries a `decode`
sub-record: the decode configuration (int8 absmax, no FWHT, M in {1, 4, 8} against
W [6912 x 2560] and [2560 x 6912], six forwards per pass) measured the same way with
its own roofline, step time and CPU baseline, and a `decode_tl2` sub-record: the same
decode configuration with the weights in the TL2 format (5 bits per 3 weights).
Inputs are seeded synthetic tensors.

Timing: W untimed warm-up steps, then exactly K steps, each one CUDA graph replay,
bracketed by a barrier and a device synchronisation, timed with CUDA events on the
launching stream; the maximum over ranks is reported.  Inputs larger than 4x L2
(the default workload's pass reads 660 MiB of X and packed weights), or rotated over
enough copies that every pass reads them from HBM.  Clocks are read through NVML every
2 ms during the timed region.  With N > 1 (torchrun), every rank runs its own replica of the
workload (the path has no cross-GPU exchange); value = tokens of all ranks / max
rank time.

--impl reference times the CPU oracle (single-threaded C, test infrastructure)
on the same workload, on rank 0 only, each step a bounded sample of tokens and
output columns extrapolated to the whole step.

Other workloads (--workload): decode, decode_tl2, prefill, wdown, wdown_swiglu,
msweep_M<M>, kvcache.  --out-dtype bf16 stores the forward workloads' outputs in bf16.  Besides
the contract's keys the line carries `roofline` (the dominant kernel alone, timed in
one graph over every input rotation), `act_quant` (the activation kernel alone, the
same way), `e2e`
(the public forward with pinned host buffers in and out) and `clocks`.
--probe-library-int8 prints cuBLASLt's dense int8 GEMM rate at 8192^3 instead, for
context beside the int8 roofline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary GEMM TOPS & weight GB/s vs roofline; H-BitLinear tokens/s (1 B200)"
# The largest configuration that fits one GPU: the M = 8192 point of the 4096-hidden
# M-sweep (Wo [4096 x 4096] and Wdown [4096 x 16384], int4 + FWHT), 1.37 Tera int ops
# per step.  The default run adds the decode configuration as a sub-record.
DEFAULT_WORKLOAD = "msweep_M8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
MAX_BATCHES = 512  # passes per timed step at most


# ----------------------------------------------------------------------------- workloads
def workload_cases(name: str):
    """(label, M, N, K, mode, fwht, x_kind, x_dtype, outliers) of one step of each workload."""
    if name in ("decode", "decode_tl2"):
        return [(name, M, N, K, "int8", False, "normal", "f32", 0)
                for (N, K) in ((6912, 2560), (2560, 6912)) for M in (1, 4, 8)]
    if name == "prefill":
        cases = []
        for w, N, fw in (("Wq", 4096, False), ("Wk", 4096, False), ("Wv", 4096, False), ("Wo", 4096, True),
                         ("Wup", 11008, False), ("Wgate", 11008, False)):
            cases.append((w, 4096, N, 4096, "int8", fw, "normal", "bf16", 0))
        return cases
    if name == "wdown":
        return [("wdown", 2048, 2048, 8192, "int4", True, "student_t3", "f32", 82)]
    if name == "wdown_swiglu":
        return [("wdown_swiglu", 2048, 2048, 8192, "int4", True, "swiglu", "f32", 0)]
    m = re.fullmatch(r"msweep_M(\d+)", name)
    if m:
        M = int(m.group(1))
        return [("Wo", M, 4096, 4096, "int4", True, "student_t3", "f32", 41),
                ("Wdown", M, 4096, 16384, "int4", True, "student_t3", "f32", 164)]
    raise SystemExit(f"unknown workload {name!r}")


WORKLOAD_TEXT = {
    "decode_tl2": "decode GEMV with the weights in the TL2 format (5 bits per 3 weights, mirror-consolidated triplets "
                  "of the edge page): int8 absmax, no FWHT, X fp32 [M,K] N(0,1), M in {1,4,8}, W [6912x2560] and "
                  "[2560x6912]; 6 forwards per step",
    "decode": "decode GEMV, int8 absmax, no FWHT: X fp32 [M,K] N(0,1), M in {1,4,8}, against ternary W "
              "[6912x2560] and [2560x6912] (N(0,0.02) absmean-ternarised, 2-bit packed); 6 forwards per step",
    "prefill": "prefill int8, 7B-like projections: X bf16 [4096,4096]; W Wq/Wk/Wv/Wo [4096x4096] (FWHT on Wo only) "
               "and Wup/Wgate [11008x4096]; 6 forwards per step",
    "wdown_swiglu": "FFN down projection fused with its SwiGLU input: gate N(0,2^2) and up N(0,1) [2048,8192] "
                    "-> silu(gate)*up formed in the activation kernel -> int4 absmean + FWHT; W [2048x8192]",
    "wdown": "Wdown-style H-BitLinear, int4 absmean + FWHT: X Student-t(3) [2048,8192] with 1% channels x50; "
             "W [2048x8192]",
}


def workload_text(name):
    if name in WORKLOAD_TEXT:
        return WORKLOAD_TEXT[name]
    return f"M-sweep point ({name}): int4 + FWHT, Student-t(3) X with 1% outlier channels x50; Wo [4096x4096] " \
           f"and Wdown [4096x16384]"


def _xdt_name(c):
    """"bf16" or "f32": the storage type of a case's X."""
    return "bf16" if str(c.X.dtype) == "torch.bfloat16" else "f32"


def make_inputs(cases, seed=0):
    """Host tensors (X, W) for every case, drawn from the shared synthetic generators."""
    from ternary_weight_bit_b200 import synthetic
    out = []
    for i, (label, M, N, K, mode, fwht, xk, xdt, outl) in enumerate(cases):
        c = synthetic.make_case(label, M, K, N, x_kind=xk, outliers=outl, outlier_gain=50.0 if outl else 20.0,
                                x_dtype=xdt, fwht=fwht, mode=mode, seed=seed + i)
        out.append(c)
    return out


def algorithmic_bytes(M, N, K, xdt, out_bytes=4, weight_bytes=None):
    """Bytes the method must move per forward: X in, codes/scales round trip, packed W (2 bits per
    weight unless weight_bytes says otherwise), fp32 (or bf16) out."""
    xb = 2 if xdt == "bf16" else 4
    wb = N * K // 4 if weight_bytes is None else weight_bytes
    act = M * K * xb + M * K + 4 * M            # act_quant: read X, write codes + scale
    gemm = wb + M * K + 4 * M + out_bytes * M * N + 4  # packed W, codes, scales, out, alpha
    return act, gemm


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profile_traffic(kernel_key: str, source_file: str):
    """Per-launch DRAM bytes of the dominant kernel on this workload, from the committed ncu
    summary profiles/<kernel_key>.md, if the kernel source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", f"{kernel_key}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m1 = re.search(r"traffic_bytes_per_launch\s*=\s*([0-9.eE+]+)", text)
    m2 = re.search(r"source_sha256\s*=\s*([0-9a-f]{64})", text)
    if not (m1 and m2):
        return None
    src = open(os.path.join(ROOT, "ternary_weight_bit_b200", "csrc", source_file), "rb").read()
    if hashlib.sha256(src).hexdigest() != m2.group(1):
        return None
    return float(m1.group(1))


# ----------------------------------------------------------------------------- clocks
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML every `period_s` from a host
    thread (reading only; nothing is set).  A timed region of a few tens of
    milliseconds still collects tens of samples this way."""

    def __init__(self, uuid: str, period_s: float = 0.002):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.period = period_s
        self.samples = []
        self._stop = threading.Event()
        self.thread = None
        get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        self._reasons = get
        self._bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                      pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)

    def start(self):
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = int(self._reasons(self.h))
                self.samples.append((time.time(), mhz, r))
            except Exception:  # a failed read is skipped, not fatal
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0,
                    "source": "nvml"}
        reasons = sorted({REASON_NAMES[i] for (_, _, r) in inside for i, b in enumerate(self._bits) if r & b})
        return {"sm_mhz": statistics.median(m for (_, m, _) in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "source": "nvml"}


class SmiClockSampler:
    """Fallback: nvidia-smi sampling of SM clock and throttle reasons while the GPU works."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [p for (t, p) in self.samples if t0 <= t <= t1] or [p for (_, p) in self.samples]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0, "source": "smi"}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[0]) for p in inside if num(p[0]) is not None]
        mx = [num(p[1]) for p in inside if num(p[1]) is not None]
        reasons = sorted({REASON_NAMES[i] for p in inside for i in range(4) if p[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "source": "smi"}


def clock_sampler(props):
    """NVML sampler for this device (by UUID), else the nvidia-smi one."""
    uuid = ""
    try:
        uuid = str(props.uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        pass
    try:
        return NvmlClockSampler(uuid)
    except Exception:
        return SmiClockSampler(uuid)


# ----------------------------------------------------------------------------- distributed
def dist_setup(want_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def aggregate(elapsed_ms: float, tokens: float, world: int, backend_device=None):
    """Max of the per-rank times and sum of the per-rank tokens (rank 0's view)."""
    if world == 1:
        return elapsed_ms, tokens
    import torch
    import torch.distributed as dist
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=backend_device)
    n = torch.tensor([tokens], dtype=torch.float64, device=backend_device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), float(n.item())


# ----------------------------------------------------------------------------- CPU oracle timing
def time_oracle(cases, budget_s: float, steps: int | None = None, bf16_out: bool = False):
    """Time the oracle on a bounded sample of the workload.  Each case runs act_quant on
    a sample of its tokens and the integer GEMM of those tokens on a sample of output
    columns; the time is extrapolated to all M tokens and N columns.  The samples are
    sized so that one step costs about budget_s / max(steps, 4) seconds.  Returns
    (tokens/s, description, steps, seconds per step)."""
    import numpy as np
    from oracle import ref
    totals = []
    done = 0
    t_begin = time.perf_counter()
    host = make_inputs(cases)
    packs = []
    tl2 = [c.name.endswith("_tl2") for c in host]
    for c, is_tl2 in zip(host, tl2):
        packed, alpha, t = ref.pack_weights(c.W.numpy(), eps=c.eps)
        packs.append((ref.pack_tl2(t) if is_tl2 else packed, alpha))
    target_step = budget_s / max(4, steps or 4)
    elem_rate = 4e7   # rough single-core rate of the oracle's act_quant (elements/s)
    mac_rate = 2.5e8  # rough single-core rate of the packed-weight loop (MAC/s)
    row_frac = min(1.0, 0.5 * target_step * elem_rate / max(sum(c.M * c.K for c in host), 1))
    rows = [max(1, min(c.M, int(math.ceil(c.M * row_frac)))) for c in host]
    macs = sum(m * c.N * c.K for m, c in zip(rows, host))
    frac = min(1.0, 0.5 * target_step * mac_rate / max(macs, 1))
    # at least 8 columns, so that the call overhead stays small against the sampled work
    cols = [max(min(c.N, 8), min(c.N, int(math.ceil(c.N * frac)))) for c in host]
    # the dequant epilogue costs per output element: it runs on the full width of the
    # sampled tokens (on zero sums), so only the integer GEMM is extrapolated over columns
    acc_full = [np.zeros((m, c.N), np.int32) for m, c in zip(rows, host)]
    while True:
        t_step = 0.0
        for c, m, ncols, af, (packed, alpha) in zip(host, rows, cols, acc_full, packs):
            mode = ref.ACT_INT8 if c.mode == "int8" else ref.ACT_INT4
            X = c.X[:m].float().numpy()
            t0 = time.perf_counter()
            if c.up is not None:
                X = ref.swiglu(X, c.up[:m].float().numpy())
            q, s_ = ref.act_quant(X, None, c.eps, c.fwht, mode)
            t1 = time.perf_counter()
            if c.name.endswith("_tl2"):
                ref.gemm_tl2(q, packed[:ncols], ncols)
            else:
                ref.gemm_packed(q, packed[:ncols], ncols)
            t2 = time.perf_counter()
            o = ref.dequant(af, s_, alpha, mode)
            if bf16_out:
                ref.round_bf16(o)
            t3 = time.perf_counter()
            t_step += ((t1 - t0) + (t2 - t1) * (c.N / ncols) + (t3 - t2)) * (c.M / m)
        totals.append(t_step)
        done += 1
        elapsed = time.perf_counter() - t_begin
        if steps is not None and done >= steps:
            break
        if steps is None and (elapsed >= budget_s or done >= 50):
            break
    tokens = sum(c.M for c in host)
    per_step = statistics.median(totals)
    sampled_rows = sum(rows)
    desc = (f"oracle (single-threaded C) on the same inputs: act_quant on {sampled_rows} of {tokens} tokens, "
            f"their integer GEMM on {sum(cols)} of {sum(c.N for c in host)} output columns, extrapolated to all "
            f"tokens and columns; "
            f"{done} step(s), median")
    return tokens / per_step, desc, done, per_step


# ----------------------------------------------------------------------------- GPU arm
def batches_per_step(pass_ms: float, min_step_ms: float) -> int:
    """Passes per timed step: enough for min_step_ms of device time, 1..MAX_BATCHES."""
    return int(max(1, min(MAX_BATCHES, math.ceil(min_step_ms / max(pass_ms, 1e-3)))))


def _timed_graph_replays(torch, graph, stream, min_s: float, max_reps: int = 100000):
    """Replay `graph` on `stream` for at least min_s seconds (3 untimed replays first);
    returns (milliseconds, replays), timed with CUDA events on that stream."""
    with torch.cuda.stream(stream):
        for _ in range(3):
            graph.replay()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        graph.replay()
    e1.record(stream)
    e1.synchronize()
    one = max(e0.elapsed_time(e1), 1e-3)
    reps = int(max(3, min(max_reps, math.ceil(min_s * 1e3 / one))))
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            graph.replay()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1), reps


def measure_forward(torch, tb, name, dev, world, steps, warmup, bf16_out, sampler, stream, sub_s=0.4, e2e=True,
                    min_step_ms=5.0):
    """One forward workload on this rank: the timed steps (CUDA graphs, events on the
    launching stream), then the dominant kernel alone, the activation kernel alone and
    the end-to-end public call.  Returns the rank-local figures."""
    cases = workload_cases(name)
    host = make_inputs(cases)
    tl2 = name.endswith("_tl2")
    if tl2 and bf16_out:
        raise SystemExit("--out-dtype bf16 applies to the 2-bit workloads")
    if bf16_out and any(c.up is not None for c in host):
        raise SystemExit("--out-dtype bf16 applies to the plain forward workloads")
    out_dtype = torch.bfloat16 if bf16_out else torch.float32
    out_bytes = 2 if bf16_out else 4
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)

    # pack once per weight matrix (offline step, not timed)
    base = []
    for c in host:
        W = c.W.to(dev)
        packed, alpha = tb.bitnet_pack_ternary(W, eps=c.eps)
        del W
        base.append((tb.bitnet_pack_tl2(packed, c.K) if tl2 else packed, alpha))
    packed_bytes = sum(p.numel() for p, _ in base)

    def in_bytes(c):
        return c.X.numel() * c.X.element_size() * (2 if c.up is not None else 1)

    step_bytes = packed_bytes + sum(in_bytes(c) for c in host)
    R = max(1, min(64, math.ceil(4 * l2 / step_bytes))) if step_bytes < 4 * l2 else 1
    rot = []  # R copies of (X, packed, alpha, out, ws, up) per case
    for r in range(R):
        items = []
        for c, (p, a) in zip(host, base):
            X = c.X.to(dev)
            U = None if c.up is None else c.up.to(dev)
            ws = torch.empty((max(tb.bitnet_forward_workspace_bytes(c.M, c.K), 256),), dtype=torch.uint8,
                             device=dev)
            out = torch.empty((c.M, c.N), dtype=out_dtype, device=dev)
            items.append((X, p.clone() if r else p, a, out, ws, U))
        rot.append(items)
    torch.cuda.synchronize()

    def forward(c, X, p, a, out, ws, U):
        if tl2:
            tb.bitnet_hbitlinear_forward_tl2(X, p, a, c.N, eps=c.eps, fwht=c.fwht, mode=c.mode, out=out, ws=ws)
        elif U is None and bf16_out:
            tb.bitnet_hbitlinear_forward_ex(X, p, a, c.N, eps=c.eps, fwht=c.fwht, mode=c.mode,
                                            out_dtype=torch.bfloat16, out=out, ws=ws)
        elif U is None:
            tb.bitnet_hbitlinear_forward(X, p, a, c.N, eps=c.eps, fwht=c.fwht, mode=c.mode, out=out, ws=ws)
        else:
            tb.bitnet_hbitlinear_forward_swiglu(X, U, p, a, c.N, eps=c.eps, fwht=c.fwht, mode=c.mode, out=out,
                                                ws=ws)

    def step(r):
        for c, item in zip(host, rot[r]):
            forward(c, *item)

    with torch.cuda.stream(stream):
        for i in range(max(1, min(warmup, R))):
            step(i % R)  # eager warm-up also primes the per-device attribute caches
    stream.synchronize()
    # One pass = every case once on one rotation of the inputs.  A timed step is `batches`
    # passes (rotations in turn) captured in one CUDA graph, enough for MIN_STEP_MS of
    # device time, so that a few timed steps still span tens of clock samples.
    ones = []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(r)
        ones.append(g)
    with torch.cuda.stream(stream):
        for r in range(R):
            ones[r].replay()
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    with torch.cuda.stream(stream):
        for r in range(R):
            ones[r].replay()
    p1.record(stream)
    p1.synchronize()
    batches = batches_per_step(p0.elapsed_time(p1) / R, min_step_ms)
    del ones
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph, stream=stream):
        for b in range(batches):
            step(b % R)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            step_graph.replay()
    stream.synchronize()
    assert tb.bitnet_get_last_device_status(stream) == 0

    # ------------------------------------------------------------------ timed region
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(steps):
            step_graph.replay()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    elapsed = e0.elapsed_time(e1)
    clocks = sampler.summary(t_wall0, t_wall1) if sampler is not None else None
    status = tb.bitnet_get_last_device_status(stream)
    tokens_rank = steps * batches * sum(c.M for c in host)
    kernels_per_step = batches * sum(tb.bitnet_forward_kernel_count(c.M, c.N, c.K, c.fwht) for c in host)

    # ------------------------------------------------------------------ dominant kernel alone
    peaks, peak_src = load_peaks()
    decode_like = max(c.M for c in host) <= 16
    codes_scales = []
    for c, (X, p, a, out, ws, U) in zip(host, rot[0]):
        if U is None:
            codes, scale = tb.bitnet_act_quant(X, eps=c.eps, fwht=c.fwht, mode=c.mode)
        else:
            codes, scale = tb.bitnet_act_quant_swiglu(X, U, eps=c.eps, fwht=c.fwht, mode=c.mode)
        codes_scales.append((codes, scale))
    torch.cuda.synchronize(dev)

    def gemm_pass(r):
        for c, (codes, scale), (X, p, a, out, ws, U) in zip(host, codes_scales, rot[r]):
            if tl2:
                tb.bitnet_ternary_gemm_tl2(codes, scale, c.mode, p, a, c.N, out=out)
            elif bf16_out:
                tb.bitnet_ternary_gemm_ex(codes, scale, c.mode, p, a, c.N, out_dtype=torch.bfloat16, out=out)
            else:
                tb.bitnet_ternary_gemm(codes, scale, c.mode, p, a, c.N, out=out)

    gg = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        gemm_pass(0)
    stream.synchronize()
    with torch.cuda.graph(gg, stream=stream):
        for r in range(R):
            gemm_pass(r)
    gemm_ms, reps = _timed_graph_replays(torch, gg, stream, sub_s)
    launches = reps * R * len(host)
    gemm_bytes = reps * R * sum(algorithmic_bytes(c.M, c.N, c.K, "f32", out_bytes, p.numel())[1]
                                for c, (p, _) in zip(host, base))
    gemm_ops = reps * R * sum(2.0 * c.M * c.N * c.K for c in host)
    weight_bytes = reps * R * sum(p.numel() for p, _ in base)
    avg_launch_s = gemm_ms / 1e3 / launches
    if decode_like:
        achieved = gemm_bytes / launches / avg_launch_s / 1e9
        peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": profile_traffic(f"gemv_traffic_{name}", "tl2.cu" if tl2 else "gemv.cu"),
                "kernel": ("gemv_tl2_kernel (TL2 triplets decoded through a 32-entry shared-memory table, mma.sync s8)"
                           if tl2 else "gemv_kernel (register-streamed packed weights, mma.sync s8, in-CTA split-K)"),
                "peak_source": f"hbm_gbs of {peak_src} MEASURED_PEAKS.json (copy, burst)",
                "avg_launch_us": round(avg_launch_s * 1e6, 3),
                "bytes_per_launch": round(gemm_bytes / launches)}
    else:
        achieved = gemm_ops / launches / avg_launch_s / 1e12
        bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak = 2.0 * bf16
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "traffic": profile_traffic(f"gemm_tc_traffic_{name}", "gemm_sm100.cu"),
                "kernel": "gemm_tc_kernel (tcgen05 kind::i8, weights as TMEM A operand, TMEM accumulator)",
                "peak_source": f"int8 dense = 2 x bf16_tflops of {peak_src} MEASURED_PEAKS.json (nominal ratio)",
                "avg_launch_us": round(avg_launch_s * 1e6, 3),
                "ops_per_launch": round(gemm_ops / launches)}

    # ------------------------------------------------------------------ activation kernel alone
    # (rows RMSNorm / FWHT / quantise): one graph over every case and rotation, into the
    # codes and scales above; algorithmic bytes = X (and up) in, codes and scales out
    def act_pass(r):
        for c, (codes, scale), (X, p, a, out, ws, U) in zip(host, codes_scales, rot[r]):
            if U is None:
                tb.bitnet_act_quant(X, eps=c.eps, fwht=c.fwht, mode=c.mode, codes=codes, scale_x=scale)
            else:
                tb.bitnet_act_quant_swiglu(X, U, eps=c.eps, fwht=c.fwht, mode=c.mode, codes=codes, scale_x=scale)

    ga = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ga, stream=stream):
        for r in range(R):
            act_pass(r)
    a_ms, a_reps = _timed_graph_replays(torch, ga, stream, sub_s)
    act_s = a_ms / 1e3 / (a_reps * R * len(host))
    act_bytes = sum(in_bytes(c) + c.M * c.K + 4 * c.M for c in host) / len(host)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    act = {"kernel": "act_quant (RMSNorm, FWHT when on, int8/int4 codes)", "bound": "hbm",
           "avg_launch_us": round(act_s * 1e6, 3), "bytes_per_launch": round(act_bytes),
           "achieved": round(act_bytes / act_s / 1e9, 1), "peak": hbm, "unit": "GB/s",
           "frac": round(act_bytes / act_s / 1e9 / hbm, 4)}

    # ------------------------------------------------------------------ end to end through the public API
    e2e_res = None
    if e2e:
        pinned_x = [c.X.pin_memory() for c in host]
        pinned_u = [None if c.up is None else c.up.pin_memory() for c in host]
        pinned_o = [torch.empty((c.M, c.N), dtype=out_dtype).pin_memory() for c in host]

        def e2e_step(i):
            for c, hx, hu, ho, (X, p, a, out, ws, U) in zip(host, pinned_x, pinned_u, pinned_o, rot[i % R]):
                X.copy_(hx, non_blocking=True)
                if U is not None:
                    U.copy_(hu, non_blocking=True)
                forward(c, X, p, a, out, ws, U)
                ho.copy_(out, non_blocking=True)

        with torch.cuda.stream(stream):
            for i in range(2):
                e2e_step(i)
        stream.synchronize()
        e2e_steps = max(3, min(steps, 200))
        x0 = torch.cuda.Event(enable_timing=True)
        x1 = torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        with torch.cuda.stream(stream):
            for i in range(e2e_steps):
                e2e_step(i)
        x1.record(stream)
        x1.synchronize()
        e2e_max, e2e_tokens = aggregate(x0.elapsed_time(x1), e2e_steps * sum(c.M for c in host), world, dev)
        e2e_res = {"value": round(e2e_tokens / (e2e_max / 1e3), 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": sum(in_bytes(c) for c in host),
                   "d2h_bytes_per_step": sum(out_bytes * c.M * c.N for c in host),
                   "note": "eager calls of the public forward with pinned host inputs in and output out per step"}
    del step_graph
    return {"cases": cases, "host": host, "R": R, "batches": batches, "step_bytes": step_bytes, "elapsed_ms": elapsed,
            "tokens_rank": tokens_rank, "clocks": clocks, "status": status, "roofline": roof,
            "act_quant": act,
            "gemm_tops": round(gemm_ops / (gemm_ms / 1e3) / 1e12, 3),
            "weight_gbs": round(weight_bytes / (gemm_ms / 1e3) / 1e9, 1), "e2e": e2e_res,
            "gpu_launches": steps * kernels_per_step}


def run_ours(args):
    import torch
    import ternary_weight_bit_b200 as tb

    world, rank, local = dist_setup(args.gpus)
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    bf16_out = args.out_dtype == "bf16"
    props = torch.cuda.get_device_properties(dev)
    sampler = clock_sampler(props)
    sampler.start()
    time.sleep(0.05)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream(dev))

    m = measure_forward(torch, tb, args.workload, dev, world, args.steps, args.warmup, bf16_out, sampler, stream)
    max_ms, tokens_all = aggregate(m["elapsed_ms"], m["tokens_rank"], world, dev)
    sub = sub_tl2 = None
    if args.workload == DEFAULT_WORKLOAD and not args.no_decode_record:
        # the decode configuration, same rules (steps of at least 5 ms), in the same process
        d_steps = args.steps
        d = measure_forward(torch, tb, "decode", dev, world, d_steps, args.warmup, bf16_out, sampler, stream,
                            e2e=False)
        d_ms, d_tok = aggregate(d["elapsed_ms"], d["tokens_rank"], world, dev)
        sub = {"workload": workload_text("decode"), "name": "decode", "steps": d_steps, "warmup": args.warmup,
               "value": round(d_tok / (d_ms / 1e3), 1), "unit": "tokens/s",
               "ms_per_step": round(d_ms / d_steps, 6), "batches_per_step": d["batches"],
               "roofline": d["roofline"], "act_quant": d["act_quant"], "gpu_launches": d["gpu_launches"],
               "clocks": {k: d["clocks"][k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
               "device_status": d["status"]}
        # the same decode configuration with the weights in the TL2 format
        t = measure_forward(torch, tb, "decode_tl2", dev, world, d_steps, args.warmup, False, sampler, stream,
                            e2e=False)
        t_ms, t_tok = aggregate(t["elapsed_ms"], t["tokens_rank"], world, dev)
        sub_tl2 = {"workload": workload_text("decode_tl2"), "name": "decode_tl2", "steps": d_steps,
                   "value": round(t_tok / (t_ms / 1e3), 1), "unit": "tokens/s",
                   "ms_per_step": round(t_ms / d_steps, 6), "batches_per_step": t["batches"],
                   "roofline": t["roofline"],
                   "gpu_launches": t["gpu_launches"], "device_status": t["status"]}
    sampler.stop()

    result = None
    if rank == 0:
        value = tokens_all / (max_ms / 1e3)
        R, step_bytes = m["R"], m["step_bytes"]
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": workload_text(args.workload), "name": args.workload,
                       "batches_per_step": m["batches"],
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs rotate over {R} copies ({R * step_bytes / 2**20:.0f} MiB > 4x L2)"
                       if R > 1 else f"per-pass working set {step_bytes / 2**20:.0f} MiB, larger than 4x L2",
                       "cuda_graphs": True, "pdl": True, "out_dtype": args.out_dtype},
            "roofline": m["roofline"],
            "act_quant": m["act_quant"],
            "gemm_tops": m["gemm_tops"],
            "weight_gbs": m["weight_gbs"],
            "e2e": m["e2e"],
            "gpu_launches": m["gpu_launches"],
            "clocks": {k: m["clocks"][k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples", "source")},
            "device_status": m["status"],
        }
        if sub is not None:
            result["decode"] = sub
        if sub_tl2 is not None:
            result["decode_tl2"] = sub_tl2
    # every rank has finished its GPU work; rank 0 now times the oracle on the host (N=1 only)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            v, desc, n, per_step = time_oracle(m["cases"], budget_s=args.cpu_budget, bf16_out=bf16_out)
            result["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                      "sample": desc}
            if sub is not None:
                v, desc, n, per_step = time_oracle(workload_cases("decode"), budget_s=max(3.0, args.cpu_budget / 3),
                                                   bf16_out=bf16_out)
                result["decode"]["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": 1,
                                                    "kind": "oracle", "sample": desc}
        print(json.dumps(result), flush=True)


# ----------------------------------------------------------------------------- KV-cache workload
KV_SHAPE = (1, 32, 4096, 128)  # B, H, S, D: one layer's keys (and values) over a 4096-token context
KV_BITS = 4
KV_TEXT = ("low-bit KV cache (BitNetV2Attention._quantize_kv_head): K and V [1, 32, 4096, 128] fp32, Student-t(3) "
           "with every 16th channel x6; token 0 int8, the rest int4 absmean; codes int8 + per-row step")


def kv_inputs(seed=0):
    from ternary_weight_bit_b200 import synthetic
    gen = synthetic.generator(seed)
    out = []
    for _ in range(2):  # K, then V
        t = synthetic.student_t3(KV_SHAPE, gen)
        t[..., ::16] *= 6.0
        out.append(t)
    return out


def time_oracle_kv(budget_s: float, steps: int | None = None):
    """The oracle kv_quant on a sample of heads, extrapolated to all heads of K and V."""
    import numpy as np
    from oracle import ref
    K, V = kv_inputs()
    B, H, S, D = KV_SHAPE
    heads = 1
    totals = []
    t_begin = time.perf_counter()
    while True:
        t = 0.0
        for T in (K, V):
            x = np.ascontiguousarray(T[:, :heads].numpy())
            t0 = time.perf_counter()
            ref.kv_quant(x, KV_BITS)
            t += (time.perf_counter() - t0) * (H / heads)
        totals.append(t)
        if steps is not None and len(totals) >= steps:
            break
        if steps is None and (time.perf_counter() - t_begin >= budget_s or len(totals) >= 50):
            break
    per_step = statistics.median(totals)
    desc = (f"oracle (single-threaded C) kv_quant on {heads} of {H} heads of K and V, extrapolated to all heads; "
            f"{len(totals)} step(s), median")
    return B * S / per_step, desc, per_step


def run_kv(args):
    import torch
    import ternary_weight_bit_b200 as tb

    world, rank, local = dist_setup(args.gpus)
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    host = kv_inputs()
    B, H, S, D = KV_SHAPE
    in_bytes = sum(t.numel() * 4 for t in host)
    R = max(2, math.ceil(4 * l2 / in_bytes))
    rot = []
    for r in range(R):
        rot.append([(t.to(dev), torch.empty(KV_SHAPE, dtype=torch.int8, device=dev),
                     torch.empty(KV_SHAPE[:-1], dtype=torch.float32, device=dev)) for t in host])
    torch.cuda.synchronize()

    def step(r):
        for x, codes, st in rot[r]:
            tb.bitnet_kv_quant(x, bits=KV_BITS, codes=codes, step=st)

    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(stream):
        for i in range(max(1, min(args.warmup, R))):
            step(i % R)
    stream.synchronize()
    # a timed step is `batches` passes (rotations in turn) in one graph, at least 5 ms
    one = torch.cuda.CUDAGraph()
    with torch.cuda.graph(one, stream=stream):
        for r in range(R):
            step(r)
    with torch.cuda.stream(stream):
        one.replay()
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    with torch.cuda.stream(stream):
        one.replay()
    p1.record(stream)
    p1.synchronize()
    batches = batches_per_step(p0.elapsed_time(p1) / R, 5.0)
    del one
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph, stream=stream):
        for b in range(batches):
            step(b % R)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step_graph.replay()
    stream.synchronize()
    sampler = clock_sampler(props)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            step_graph.replay()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    elapsed = e0.elapsed_time(e1)
    max_ms, tokens_all = aggregate(elapsed, args.steps * batches * B * S, world, dev)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    status = tb.bitnet_get_last_device_status(stream)
    # the kernel alone: one graph over every rotation, replayed, so that graph-launch
    # gaps between steps do not count against the launch duration
    gg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gg, stream=stream):
        for r in range(R):
            step(r)
    reps = max(3, min(200, int(400 / R)))
    with torch.cuda.stream(stream):
        for _ in range(3):
            gg.replay()
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    k0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            gg.replay()
    k1.record(stream)
    k1.synchronize()
    launches = reps * R * 2  # two launches (K, V) per step
    avg_launch_s = k0.elapsed_time(k1) / 1e3 / launches
    bytes_per_launch = B * H * S * (4 * D + D + 4)  # read fp32, write int8 codes and the fp32 step
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = bytes_per_launch / avg_launch_s / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": profile_traffic("kv_quant_traffic_kvcache", "kv_quant.cu"),
            "kernel": "kv_quant_kernel (a warp per group of (b, h, s) rows, 16-byte loads, shuffle reductions)",
            "peak_source": f"hbm_gbs of {peak_src} MEASURED_PEAKS.json (copy, burst)",
            "avg_launch_us": round(avg_launch_s * 1e6, 3), "bytes_per_launch": bytes_per_launch}
    # end to end through the public API: H2D of K and V, quantise, D2H of codes and steps
    pin_in = [t.pin_memory() for t in host]
    pin_c = [torch.empty(KV_SHAPE, dtype=torch.int8).pin_memory() for _ in host]
    pin_s = [torch.empty(KV_SHAPE[:-1], dtype=torch.float32).pin_memory() for _ in host]
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_once(r):
        for hi, hc, hs, (x, codes, st) in zip(pin_in, pin_c, pin_s, rot[r]):
            x.copy_(hi, non_blocking=True)
            tb.bitnet_kv_quant(x, bits=KV_BITS, codes=codes, step=st)
            hc.copy_(codes, non_blocking=True)
            hs.copy_(st, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_once(0)
    stream.synchronize()
    x0 = torch.cuda.Event(enable_timing=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(e2e_steps):
            e2e_once(i % R)
    x1.record(stream)
    x1.synchronize()
    e2e_max, e2e_tokens = aggregate(x0.elapsed_time(x1), e2e_steps * B * S, world, dev)
    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": round(tokens_all / (max_ms / 1e3), 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 6),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": KV_TEXT, "name": "kvcache", "batches_per_step": batches,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs rotate over {R} copies ({R * in_bytes / 2**20:.0f} MiB > 4x L2)",
                       "cuda_graphs": True, "pdl": True},
            "roofline": roof,
            "e2e": {"value": round(e2e_tokens / (e2e_max / 1e3), 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": sum(c.numel() + 4 * s.numel()
                                                                               for c, s in zip(pin_c, pin_s)),
                    "note": "eager bitnet_kv_quant calls with pinned host K, V in and codes, steps out per step"},
            "gpu_launches": 2 * batches * args.steps,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples", "source")},
            "device_status": status,
        }
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            v, desc, _ = time_oracle_kv(budget_s=args.cpu_budget)
            result["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                      "sample": desc}
        print(json.dumps(result), flush=True)


def run_reference(args):
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    if args.workload == "kvcache":
        budget = max(10.0, min(150.0, 6.0 * (args.steps + args.warmup)))
        if args.warmup:
            time_oracle_kv(budget, steps=1)
        v, desc, per_step = time_oracle_kv(budget, steps=args.steps)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": KV_TEXT, "name": "kvcache"},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return
    cases = workload_cases(args.workload)
    budget = max(10.0, min(150.0, 6.0 * (args.steps + args.warmup)))
    # warm-up steps are untimed samples too; time exactly --steps steps
    bf16_out = args.out_dtype == "bf16"
    if args.warmup:
        time_oracle(cases, budget_s=budget, steps=1, bf16_out=bf16_out)
    v, desc, n, per_step = time_oracle(cases, budget_s=budget, steps=args.steps, bf16_out=bf16_out)
    tokens = sum(c[1] for c in cases)
    result = {
        "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": workload_text(args.workload), "name": args.workload, "out_dtype": args.out_dtype},
        "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": f"{tokens} tokens per step",
    }
    print(json.dumps(result), flush=True)


def run_library_int8_probe(args):
    """Context only, not a bench line: the dense int8 GEMM rate torch._int_mm (cuBLASLt) reaches on
    this GPU at 8192^3, beside the nominal-ratio int8 peak the roofline divides by."""
    import torch
    dev = torch.device("cuda", 0)
    n = 8192
    a = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=dev)
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = 20
    e0.record()
    for _ in range(reps):
        torch._int_mm(a, b)
    e1.record()
    e1.synchronize()
    s_ = e0.elapsed_time(e1) / 1e3 / reps
    peaks, src = load_peaks()
    print(json.dumps({"probe": "torch._int_mm int8 8192^3 (library GEMM, context)", "tops": round(2 * n ** 3 / s_ / 1e12, 1),
                      "ms_per_gemm": round(s_ * 1e3, 3),
                      "nominal_int8_peak_tops": round(2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])), 1),
                      "peak_source": src}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help=f"{DEFAULT_WORKLOAD} (default) | decode | decode_tl2 | prefill | wdown | wdown_swiglu | "
                         "msweep_M<M> | kvcache")
    ap.add_argument("--no-decode-record", action="store_true",
                    help="skip the decode sub-record of the default workload")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--out-dtype", choices=["f32", "bf16"], default="f32",
                    help="output storage of the forward workloads: fp32, or bf16 rounded to nearest even")
    ap.add_argument("--probe-library-int8", action="store_true",
                    help="print the rate of torch._int_mm at 8192^3 (context for the int8 roofline) and exit")
    args = ap.parse_args()
    if args.probe_library_int8:
        run_library_int8_probe(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "kvcache":
        run_kv(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
