"""Benchmark of the routed mixture-of-experts layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|skewed]
                    [--impl native|reference]

One step = one pass of the whole layer (router, top-K, permute, row gather,
up GEMM + ReLU^2, down GEMM, combine) over one batch of seeded synthetic
tokens, through the C ABI's moe_forward.  The default workload is the
decode-sized layer (64 tokens, hidden 2688, 128 experts, top-6, expert width
1856, bf16); a prefill-chunk (4096-token) measurement is reported beside it.

Under torchrun (N > 1) every rank runs its own batch on its own GPU with
replicated weights (the layer is independent per token): weak scaling, no
data-path collective; the time is the max over ranks.

Prints ONE JSON line on rank 0.  ``--impl reference`` times the CPU oracle
(the plain fp64 statement of the layer) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "MoE-layer tokens/s on 1 B200; % of HBM roofline (decode), % TC peak (prefill)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {"tiny": 0, "decode": 1, "prefill": 2, "skewed": 3, "chain": 4, "decode_nvfp4": 5,
             "prefill_nvfp4": 6, "decode_shared": 7, "prefill_shared": 8, "decode_fp8_b128": 9,
             "prefill_fp8_b128": 10}
L2_WARM_BYTES = 48 << 20   # the library's default L2 prefetch of a bf16 up bank at small batches
TENSOR_BOUND = ("prefill", "chain", "prefill_nvfp4", "prefill_shared",
                "prefill_fp8_b128")   # reported against the tensor peak


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def reduce_max(value: float, dist=None, device=None) -> float:
    """Max over ranks (identity on one rank): every multi-GPU time is the slowest rank's."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank: int, steps: int, ms: float) -> float:
    """Whole-job throughput: tokens processed by all ranks / the max-over-ranks time."""
    return world * tokens_per_rank * steps / (ms * 1e-3)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Clocks and throttle reasons, sampled while the timed region runs.

    Through NVML every 1-2 ms when the bindings load (a decode timed region of 20 steps lasts
    under 10 ms), in a child process so that the timed loop's thread does not starve it, else
    through `nvidia-smi -lms 100`.  Samples are stamped with the host's monotonic clock (the
    same in both processes); `window(t0, t1)` keeps those taken between the timed region's
    start and end (the bench records both around its synchronised loop), so the line's clocks
    are those under load.
    """

    # the child: one line per sample, "t, sm, max, power, reasons, hw_slowdown, hw_thermal,
    # sw_thermal, sw_power_cap" (the nvidia-smi field order after the time stamp)
    NVML_CHILD = r"""
import sys, time, pynvml as nv
nv.nvmlInit()
u = sys.argv[1]
h = nv.nvmlDeviceGetHandleByUUID(u) if u else nv.nvmlDeviceGetHandleByIndex(0)
bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
        nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
mx = str(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
print("ready", flush=True)
n = 0
pw = "0.0"
while True:
    # two queries per sample (the SM clock and the reasons); the power draw every 16th
    t = time.perf_counter()
    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
    if n % 16 == 0:
        pw = f"{nv.nvmlDeviceGetPowerUsage(h) / 1000.0:.1f}"
    n += 1
    f = ["Active" if r & b else "Not Active" for b in bits]
    print(", ".join([f"{t:.6f}", str(sm), mx, pw, hex(r)] + f), flush=True)
    time.sleep(0.001)
"""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    NVML_PERIOD_S = 0.002

    def __init__(self, gpu_uuid: str | None, nvml=None):
        self.uuid = gpu_uuid
        self.proc = None
        self.lines = []      # (host time, csv line in the nvidia-smi field order)
        self.thread = None
        self.nvml = nvml
        self.handle = None
        self.stop_flag = threading.Event()
        self.win = None
        self.stamped = False
        self.source = "nvidia-smi -lms 100"

    def _nvml_open(self):
        try:
            nv = self.nvml
            if nv is None:
                import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else nv.nvmlDeviceGetHandleByIndex(0)
            self.nvml, self.handle = nv, h
            self.source = "nvml, every 2 ms"
            return True
        except Exception:
            self.nvml = self.handle = None
            return False

    def _nvml_loop(self):
        nv, h = self.nvml, self.handle
        bits = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
                ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
                ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
                ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap")]
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                flags = ["Active" if r & getattr(nv, name) else "Not Active" for _, name in bits]
                self.lines.append((time.perf_counter(), ", ".join([str(sm), str(mx), f"{pw:.1f}", hex(r)] + flags)))
            except Exception:
                return
            time.sleep(self.NVML_PERIOD_S)

    def start(self):
        if self.nvml is not None and self._nvml_open():   # an injected NVML (tests): a thread
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", self.NVML_CHILD, self.uuid or ""],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            if self.proc.stdout.readline().strip() == "ready":
                self.source = "nvml child process, ~1 ms apart"
                self.stamped = True
                self.thread = threading.Thread(target=self._read, daemon=True)
                self.thread.start()
                return
            self.proc.kill()
            self.proc.wait(timeout=5)
        except (OSError, subprocess.TimeoutExpired):
            pass
        self.proc = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            line = line.strip()
            if self.stamped:
                t, _, rest = line.partition(",")
                try:
                    self.lines.append((float(t), rest.strip()))
                except ValueError:
                    pass
            else:
                self.lines.append((time.perf_counter(), line))

    def window(self, t0: float, t1: float):
        """Keep the summary to samples taken between t0 and t1 (host perf_counter seconds)."""
        self.win = (t0, t1)

    def stop(self):
        if self.handle is not None:
            self.stop_flag.set()
            if self.thread:
                self.thread.join(timeout=2)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return self.summary()
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return self.summary()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        if self.win is not None:
            inside = [x for x in lines if self.win[0] <= x[0] <= self.win[1]]
            if inside:
                lines = inside
            elif lines:
                # a region shorter than the sampling period: the sample nearest its middle
                mid = 0.5 * (self.win[0] + self.win[1])
                lines = [min(lines, key=lambda x: abs(x[0] - mid))]
        for _, ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "sampler": self.source}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "sampler": self.source}


# --------------------------------------------------------------------------- native arm

class Layer:
    """Device-resident weights and buffers of one workload."""

    def __init__(self, wl, device, n_batches=4):
        import torch
        import synth
        import routed_expert_moe_b200 as moe
        from synth import workloads as W

        self.wl = wl
        self.moe = moe
        self.device = device
        bf = torch.bfloat16
        stream = torch.cuda.current_stream().cuda_stream
        self.wu = torch.empty(wl.E, wl.F, wl.H, dtype=bf, device=device)
        self.wd = torch.empty(wl.E, wl.H, wl.F, dtype=bf, device=device)
        self.wr = torch.empty(wl.E, wl.H, dtype=bf, device=device)
        synth.normal_bf16_device(synth.key(wl.seed, synth.T_WUP, 0), self.wu.numel(), W.SIGMA_W,
                                 self.wu.data_ptr(), stream)
        synth.normal_bf16_device(synth.key(wl.seed, synth.T_WDOWN, 0), self.wd.numel(), W.SIGMA_W,
                                 self.wd.data_ptr(), stream)
        synth.normal_bf16_device(synth.key(wl.seed, synth.T_WR, 0), self.wr.numel(), W.SIGMA_W,
                                 self.wr.data_ptr(), stream)
        self.bias = None
        b = W.host_bias(wl)
        if b is not None:
            self.bias = torch.from_numpy(b).to(device)
        # several token batches (batch 0 is the workload's own x; others use layer ids 1..)
        self.xs = []
        for i in range(n_batches):
            x = torch.empty(wl.T, wl.H, dtype=bf, device=device)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_X, i), x.numel(), W.SIGMA_X, x.data_ptr(), stream)
            self.xs.append(x)
        self.scales = None
        if wl.nvfp4:
            # NVFP4 banks quantised on the device from the bf16 masters; static activation scales
            # from the oracle's calibration (tests/golden/nvfp4_scales.json)
            banks = []
            for src in (self.wu, self.wd):
                n, rows, Kd = src.shape
                codes = torch.empty(n, rows, Kd // 2, dtype=torch.uint8, device=device)
                block = torch.empty(n, rows, moe.nvfp4_scale_row(Kd), dtype=torch.uint8, device=device)
                tsc = torch.empty(n, dtype=torch.float32, device=device)
                moe.quantize_nvfp4(src, codes, block, tsc)
                banks.append((codes, block, tsc))
            torch.cuda.synchronize(device)
            (self.wu, self.bu, self.tu), (self.wd, self.bd, self.td) = banks
            sx, sh = W.nvfp4_scales(wl)
            self.scales = moe.nvfp4_scales(self.tu, self.td, float(sx), float(sh), self.bu, self.bd)
        if wl.fp8_b128:
            # FP8_B128 banks quantised on the device from the bf16 masters; static activation scales
            # from the oracle's calibration (tests/golden/fp8_b128_scales.json)
            banks = []
            for src in (self.wu, self.wd):
                n, rows, Kd = src.shape
                kp = moe.b128_kp(Kd)
                codes = torch.empty(n, rows, kp, dtype=torch.uint8, device=device)
                sc = torch.empty(n, rows, kp // 128, dtype=torch.float32, device=device)
                moe.quantize_fp8_b128(src, codes, sc)
                banks.append((codes, sc))
            torch.cuda.synchronize(device)
            (self.wu, self.su), (self.wd, self.sd) = banks
            sx, sh = W.fp8_b128_scales(wl)
            self.scales = moe.fp8_scales(self.su, self.sd, float(sx), float(sh))
        self.shared = None
        if wl.shared:
            # the shared expert: W_up_s [Fs][H], W_down_s [H][Fs], bf16
            su = torch.empty(wl.shared, wl.H, dtype=bf, device=device)
            sd = torch.empty(wl.H, wl.shared, dtype=bf, device=device)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_WUP_S, 0), su.numel(), W.SIGMA_W, su.data_ptr(),
                                     stream)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_WDOWN_S, 0), sd.numel(), W.SIGMA_W, sd.data_ptr(),
                                     stream)
            self.shared = (su, sd)
        self.dims = moe.dims(wl.T, wl.H, wl.E, wl.K, wl.F, nvfp4=wl.nvfp4, Fs=wl.shared, fp8_b128=wl.fp8_b128)
        self.ws = moe.alloc_workspace(self.dims, device)
        self.out = torch.empty(wl.T, wl.H, dtype=bf, device=device)
        self.idx = torch.empty(wl.T, wl.K, dtype=torch.int32, device=device)
        self.w = torch.empty(wl.T, wl.K, dtype=torch.float32, device=device)
        torch.cuda.synchronize(device)

    def step(self, i, x=None, out=None):
        self.moe.forward(self.dims, self.xs[i % len(self.xs)] if x is None else x, self.wr, self.bias, self.wu,
                         self.wd, self.out if out is None else out, self.ws, scales=self.scales, topk_idx=self.idx,
                         topk_w=self.w, shared=self.shared)

    def touched_experts(self, i):
        import torch
        self.step(i)
        torch.cuda.synchronize()
        return int(torch.unique(self.idx).numel()), int(self.idx.numel())

    def launches_per_step(self):
        """The library's kernel launches in one step (one moe_forward)."""
        return self.moe.forward_launches(self.dims)


class Chain:
    """The 23-layer W8A8 stack of the chain workload, weights made and quantised on the device."""

    def __init__(self, wl, device):
        import torch
        import synth
        import routed_expert_moe_b200 as moe
        from routed_expert_moe_b200.stack import MoeStack
        from synth import workloads as W

        self.wl = wl
        self.moe = moe
        self.device = device
        stream = torch.cuda.current_stream().cuda_stream
        self.stack = MoeStack(wl.T, wl.H, wl.E, wl.K, wl.F, fp8=True, device=device)
        wu = torch.empty(wl.E, wl.F, wl.H, dtype=torch.bfloat16, device=device)
        wd = torch.empty(wl.E, wl.H, wl.F, dtype=torch.bfloat16, device=device)
        for l, (sx, sh) in enumerate(W.chain_scales()[:wl.layers]):
            wr = torch.empty(wl.E, wl.H, dtype=torch.bfloat16, device=device)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_WR, l), wr.numel(), W.SIGMA_W, wr.data_ptr(), stream)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_WUP, l), wu.numel(), W.SIGMA_W, wu.data_ptr(), stream)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_WDOWN, l), wd.numel(), W.SIGMA_W, wd.data_ptr(),
                                     stream)
            self.stack.add_layer(wr, wu, wd, float(sx), float(sh))
        del wu, wd
        self.xs = []
        for i in range(2):
            x = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=device)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_X, i), x.numel(), W.SIGMA_X, x.data_ptr(), stream)
            self.xs.append(x)
        self.out = self.xs[0]
        self.idx = torch.empty(wl.T, wl.K, dtype=torch.int32, device=device)
        torch.cuda.synchronize(device)

    def step(self, i, x=None, out=None):
        y = self.stack.forward(self.xs[i % len(self.xs)] if x is None else x)
        self.out = y if out is None else out.copy_(y)

    def launches_per_step(self):
        """Per layer: the RMS norm, then one moe_forward."""
        return self.wl.layers * (1 + self.moe.forward_launches(self.stack.dims))

    def profile_layer(self, i):
        """one pass of layer 0, for the stage events"""
        self.stack.run_layer(0, self.xs[0], self.stack.x[1], topk_idx=self.idx)

    def touched_experts(self, i):
        import torch
        self.profile_layer(0)
        torch.cuda.synchronize()
        return int(torch.unique(self.idx).numel()), int(self.idx.numel())


def stage_profile(layer, steps, warmup):
    """Per-stage device time (ms, mean over steps) from the library's stage events."""
    import torch
    moe = layer.moe
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.STAGE_EVENTS)] for _ in range(steps)]
    one = layer.profile_layer if hasattr(layer, "profile_layer") else layer.step
    for i in range(warmup):
        one(i)
    times = [[0.0] * (moe.STAGE_EVENTS - 1) for _ in range(steps)]
    for i in range(steps):
        moe.set_stage_events(ev[i])
        one(i)
    moe.set_stage_events(None)
    torch.cuda.synchronize()
    for i in range(steps):
        for s in range(moe.STAGE_EVENTS - 1):
            times[i][s] = ev[i][s].elapsed_time(ev[i][s + 1])
    return {name: statistics.mean(t[s] for t in times) for s, name in enumerate(moe.STAGES)}


def timed_loop(layer, steps, warmup, barrier):
    import torch
    for i in range(warmup):
        layer.step(i)
    barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    timed_loop.window = (time.perf_counter(), None)
    start.record()
    for i in range(steps):
        layer.step(i)
    stop.record()
    torch.cuda.synchronize()
    timed_loop.window = (timed_loop.window[0], time.perf_counter())
    barrier()
    return start.elapsed_time(stop)


def e2e_loop(layer, steps, warmup):
    """Same metric through the public API with host buffers: every step copies its x from pinned host
    memory to the device, runs the layer and copies its output back to pinned host memory.  The copies
    run on their own streams, double-buffered, so that step i's input upload and step i-1's download
    overlap the layer's kernels (the order a serving loop would use); the timed region spans the first
    upload to the last download."""
    import torch
    wl = layer.wl
    hx = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, pin_memory=True) for _ in range(len(layer.xs))]
    for i, x in enumerate(layer.xs):
        hx[i].copy_(x.cpu())
    hout = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    dx = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=layer.device) for _ in range(2)]
    dout = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=layer.device) for _ in range(2)]
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def one(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(done[b])          # step i-2 has read dx[b]
            dx[b].copy_(hx[i % len(hx)], non_blocking=True)
            in_ready[b].record(s_in)
        compute.wait_event(in_ready[b])
        if used[b]:
            compute.wait_event(out_free[b])       # step i-2's output has left dout[b]
        layer.step(i, x=dx[b], out=dout[b])
        done[b].record(compute)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[b])
            hout[b].copy_(dout[b], non_blocking=True)
            out_free[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(compute)
    s_in.wait_event(start)
    for i in range(steps):
        one(i)
    for b in range(2):
        compute.wait_event(out_free[b])
    stop.record(compute)
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop)
    nb = wl.T * wl.H * 2
    return ms, nb, nb


# the sources that decide what the grouped GEMM kernel runs and reads: its own
# file, the shared device helpers, and the permutation that writes its schedule
TRAFFIC_SOURCES = ("routed_expert_moe_b200/csrc/grouped_gemm.cu", "routed_expert_moe_b200/csrc/common.cuh",
                   "routed_expert_moe_b200/csrc/permute.cu")


def sources_sha256(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        h.update((ROOT / rel).read_bytes())
    return h.hexdigest()


def traffic_from_profile(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's sources still hash
    to those of the captured build."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    try:
        d = json.loads(p.read_text())
    except ValueError:
        return None
    ent = d.get(f"{kernel}@{workload}")
    if not ent:
        return None
    srcs = ent.get("sources", TRAFFIC_SOURCES)
    try:
        if ent.get("source_sha256") != sources_sha256(srcs):
            return None
    except OSError:
        return None
    return ent.get("dram_bytes_per_launch")


def roofline_entry(wl, stages, touched, peaks, peak_kind, workload):
    """Roofline of the dominant kernel of the step (an expert GEMM).

    Decode is declared HBM-bound (a weight stream); prefill and the FP8 chain
    are reported against the dense tensor peak of their dtype, as the metric
    asks, with the HBM fraction of the same launch beside it.
    """
    H, F, T, K = wl.H, wl.F, wl.T, wl.K
    ns = wl.shared // F        # shared-expert chunks: F-wide experts every token passes through
    rows = T * (K + ns)
    touched = touched + ns
    fp8 = wl.fp8 or wl.fp8_b128
    es = 1 if fp8 else 2
    if "expert_ffn" in stages:
        # both projections in one launch: that launch is the dominant kernel
        return _fused_entry(wl, stages, touched, peaks, peak_kind, workload)
    up_ms, down_ms = stages["up_gemm"], stages["down_gemm"]
    kernel = "up_gemm" if up_ms >= down_ms else "down_gemm"
    ms = max(up_ms, down_ms)
    flops = 2.0 * rows * F * H
    if wl.nvfp4:
        # packed codes (half a byte per value) + one E4M3 block scale per 16 values (rows padded to 16 bytes)
        ksp = lambda k: (k // 16 + 15) // 16 * 16
        w_b = touched * F * (H / 2 + ksp(H)) if kernel == "up_gemm" else touched * H * (F / 2 + ksp(F))
        algo = (w_b + rows * (H / 2 + ksp(H)) + rows * (F / 2 + ksp(F)) if kernel == "up_gemm"
                else w_b + rows * (F / 2 + ksp(F)) + rows * H * 2)
    elif wl.fp8_b128:
        # codes padded to whole blocks of 128 along K + one fp32 scale per block
        kp = lambda k: (k + 127) // 128 * 128
        w_b = touched * F * (kp(H) + kp(H) // 128 * 4) if kernel == "up_gemm" else touched * H * (kp(F) + kp(F) // 128 * 4)
        algo = w_b + rows * H + rows * F if kernel == "up_gemm" else w_b + rows * F + rows * H * 2
    # weights of the touched experts + activations in (es bytes) + activations out
    elif kernel == "up_gemm":
        algo = touched * F * H * es + rows * H * es + rows * F * es
    else:
        algo = touched * F * H * es + rows * F * es + rows * H * 2
    hbm_peak = peaks["hbm_gbs"]
    gbs = algo / (ms * 1e-3) / 1e9
    # the GEMM is timed by events around single launches inside short steps (well under a
    # second of work): the burst peak applies, the sustained one is reported beside it
    if fp8 and peaks.get("fp8_tflops"):
        tc_peak, src = peaks["fp8_tflops"], peaks["fp8_source"]
        tc_sust = None
    else:
        # a contraction takes its own dtype's peak: the measured bf16 one times the nominal ratio
        ratio = 4.0 if wl.nvfp4 else 2.0 if fp8 else 1.0
        tc_peak = peaks["bf16_tflops"] * ratio
        src = f"{peak_kind} bf16 burst" + (" x 4 (nvfp4/bf16 nominal ratio)" if wl.nvfp4 else
                                           " x 2 (fp8/bf16 nominal ratio)" if fp8 else "")
        tc_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * ratio
    tflops = flops / (ms * 1e-3) / 1e12
    common = {"kernel": kernel, "ms_per_launch": ms, "algorithmic_bytes_per_launch": algo,
              "algorithmic_flops_per_launch": flops, "traffic": traffic_from_profile(kernel, workload),
              "hbm_gbs": gbs, "hbm_frac": gbs / hbm_peak, "tensor_tflops": tflops, "tensor_frac": tflops / tc_peak}
    if tc_sust:
        common["tensor_frac_of_sustained"] = tflops / tc_sust
    if workload in TENSOR_BOUND:
        return dict(bound="tensor", achieved=tflops, peak=tc_peak, unit="TFLOP/s", frac=tflops / tc_peak,
                    peak_source=src, **common)
    return dict(bound="hbm", achieved=gbs, peak=hbm_peak, unit="GB/s", frac=gbs / hbm_peak,
                peak_source=f"{peak_kind} hbm copy", **common)


def probe_fp8_peak(device, n=8192, reps=10):
    """Dense E4M3 GEMM throughput of this GPU (TFLOP/s, best of `reps`): cuBLASLt through
    torch._scaled_mm on n x n x n, bf16 output, unit scales.  A measurement of the peak only;
    nothing of the layer runs through it.  None when the library call is unavailable."""
    import torch
    try:
        a = torch.randn(n, n, device=device).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=device).to(torch.float8_e4m3fn).t()   # column-major operand
        one = torch.ones((), device=device, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize(device)
        best = float("inf")
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e.record()
            torch.cuda.synchronize(device)
            best = min(best, s.elapsed_time(e))
        del a, b
        torch.cuda.empty_cache()
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


def _fused_entry(wl, stages, touched, peaks, peak_kind, workload):
    """Roofline of the one-launch expert FFN (both projections): the bytes and flops of the up and
    the down projection together, over the launch's duration."""
    H, F, T, K = wl.H, wl.F, wl.T, wl.K
    rows = T * (K + wl.shared // F)    # a shared expert's Fs/F chunks add T rows each (touched counts them)
    fp8 = wl.fp8 or wl.fp8_b128
    es = 1 if fp8 else 2
    ms = stages["expert_ffn"]
    if wl.fp8_b128:
        # codes padded to whole blocks of 128 along K + one fp32 scale per block, both banks;
        # x's codes in, H's codes out and back in, bf16 Y out
        kp = lambda k: (k + 127) // 128 * 128
        algo = (touched * F * (kp(H) + kp(H) // 128 * 4) + touched * H * (kp(F) + kp(F) // 128 * 4)
                + rows * H + 2 * rows * F + rows * H * 2)
    elif wl.nvfp4:
        # packed codes (half a byte per value) + one E4M3 block scale per 16 values (rows padded
        # to 16 bytes): both banks, x's codes in, H's codes out and back in, bf16 Y out
        ksp = lambda k: (k // 16 + 15) // 16 * 16
        algo = (touched * F * (H / 2 + ksp(H)) + touched * H * (F / 2 + ksp(F)) + rows * (H / 2 + ksp(H))
                + 2 * rows * (F / 2 + ksp(F)) + rows * H * 2)
    else:
        algo = 2 * touched * F * H * es + rows * H * es + rows * F * es + rows * F * es + rows * H * 2
    flops = 2 * 2.0 * rows * F * H
    gbs = algo / (ms * 1e-3) / 1e9
    hbm_peak = peaks["hbm_gbs"]
    if fp8 and peaks.get("fp8_tflops"):
        tc_peak, src = peaks["fp8_tflops"], peaks["fp8_source"]
    else:
        ratio = 4.0 if wl.nvfp4 else 2.0 if fp8 else 1.0
        tc_peak = peaks["bf16_tflops"] * ratio
        src = f"{peak_kind} bf16 burst" + (" x 4 (nvfp4/bf16 nominal ratio)" if wl.nvfp4 else
                                           " x 2 (fp8/bf16 nominal ratio)" if fp8 else "")
    tflops = flops / (ms * 1e-3) / 1e12
    common = {"kernel": "expert_ffn (up and down projections, one launch)", "ms_per_launch": ms,
              "algorithmic_bytes_per_launch": algo, "algorithmic_flops_per_launch": flops,
              "traffic": traffic_from_profile("expert_ffn", workload), "hbm_gbs": gbs, "hbm_frac": gbs / hbm_peak,
              "tensor_tflops": tflops, "tensor_frac": tflops / tc_peak}
    if workload in TENSOR_BOUND:
        return dict(bound="tensor", achieved=tflops, peak=tc_peak, unit="TFLOP/s", frac=tflops / tc_peak,
                    peak_source=src, **common)
    # the small-batch router (T <= 256: clusters of 4 tokens when they all fit at once, else of
    # 8; 15 clusters of 8 CTAs fit a 148-SM B200) fills the clusters left over with L2 prefetches
    # of the up bank's first bytes before this launch: achieved counts every algorithmic byte, so
    # frac can pass the copy peak by up to warm / algo
    tb = 4 if (T + 3) // 4 <= 15 else 8
    bf16 = not (fp8 or wl.nvfp4)   # the library prefetches only bf16 banks
    warm = min(L2_WARM_BYTES, wl.E * F * H * 2) if bf16 and T <= 256 and (T + tb - 1) // tb < 15 else 0
    return dict(bound="hbm", achieved=gbs, peak=hbm_peak, unit="GB/s", frac=gbs / hbm_peak,
                peak_source=f"{peak_kind} hbm copy", l2_warm_bytes_before_launch=warm, **common)


def ffn_is_one_launch(moe, dims) -> bool:
    """Whether the library runs both expert projections of these dims in one launch (one launch
    fewer than with that switched off through the test hook)."""
    on = moe.forward_launches(dims)
    moe.debug_set(8, 0)
    off = moe.forward_launches(dims)
    moe.debug_set(8, 1)
    return on < off


def stage_view(stages, one_launch):
    """Stage times under their kernels' names: with the one-launch FFN the up-projection slot
    holds both projections (the down slot is the empty gap before the combine)."""
    if not one_launch:
        return stages
    out = dict(stages)
    out["expert_ffn"] = out.pop("up_gemm") + out.pop("down_gemm")
    return out


_BANKS = {}


def _host_banks(wl, layer, used, fp8):
    """Host weight banks of the used experts (input preparation, cached, never timed)."""
    import oracle
    from synth import workloads as W
    key = (wl.name, layer, tuple(used), fp8)
    if key not in _BANKS:
        wu = W.host_w_up(wl, layer, experts=used)
        wd = W.host_w_down(wl, layer, experts=used)
        _BANKS.clear()
        _BANKS[key] = (oracle.quantize_bank_fp8(wu), oracle.quantize_bank_fp8(wd)) if fp8 else (wu, wd)
    return _BANKS[key]


CPU_SAMPLE_SECONDS = 10.0   # the oracle's timed work is repeated until it reaches this


def cpu_baseline(wl, n_tokens, seed_batch=0, target_s=CPU_SAMPLE_SECONDS):
    """The oracle as it stands, on the host cores, over a bounded sample of the workload
    (the same token sample repeated until about CPU_SAMPLE_SECONDS of work)."""
    if wl.fp8:
        return cpu_baseline_fp8(wl, n_tokens, seed_batch, target_s=target_s)
    if wl.nvfp4:
        return cpu_baseline_nvfp4(wl, n_tokens, seed_batch, target_s=target_s)
    if wl.fp8_b128:
        return cpu_baseline_fp8_b128(wl, n_tokens, seed_batch, target_s=target_s)
    import oracle
    from synth import workloads as W
    x = W.host_x(wl, seed_batch)[:n_tokens]
    wr = W.host_router(wl)
    t0 = time.perf_counter()
    _, idx, _ = oracle.route(x, wr, W.host_bias(wl), wl.K)
    used = sorted(set(idx.reshape(-1).tolist()))
    slot = -__import__("numpy").ones(wl.E, dtype="int32")
    slot[used] = range(len(used))
    t_route = time.perf_counter() - t0
    wu, wd = _host_banks(wl, 0, used, False)   # generating inputs is not timed
    shared = (W.host_w_up_shared(wl), W.host_w_down_shared(wl)) if wl.shared else None
    dt, reps = 0.0, 0
    while (reps == 0 or dt < target_s) and reps < 1000:
        t0 = time.perf_counter()
        _, idx, _ = oracle.route(x, wr, W.host_bias(wl), wl.K)
        oracle.moe_layer_bf16(x, wr, W.host_bias(wl), wu, wd, wl.K, slot=slot, shared=shared)
        dt += time.perf_counter() - t0
        reps += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": reps * n_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_tokens} of the {wl.T} tokens of batch {seed_batch} ({wl.name}), full layer "
                      f"(router, top-{wl.K}, {len(used)} experts' up/ReLU^2/down in fp64, "
                      f"{'a shared expert of width %d, ' % wl.shared if wl.shared else ''}combine), "
                      f"{reps} times; {dt:.2f} s"}


def cpu_baseline_nvfp4(wl, n_tokens, seed_batch=0, target_s=CPU_SAMPLE_SECONDS):
    """The oracle's W4A4 layer (router, NVFP4 experts, combine) on a token sample."""
    import numpy as np
    import oracle
    from synth import workloads as W
    x = W.host_x(wl, seed_batch)[:n_tokens]
    wr = W.host_router(wl)
    _, idx, _ = oracle.route(x, wr, W.host_bias(wl), wl.K)
    used = sorted(set(idx.reshape(-1).tolist()))
    slot = -np.ones(wl.E, dtype=np.int32)
    slot[used] = np.arange(len(used))
    key = (wl.name, 0, tuple(used), "nvfp4")
    if key not in _BANKS:   # weight preparation: untimed
        _BANKS.clear()
        _BANKS[key] = (oracle.quantize_bank_nvfp4(W.host_w_up(wl, experts=used)),
                       oracle.quantize_bank_nvfp4(W.host_w_down(wl, experts=used)))
    bank_up, bank_down = _BANKS[key]
    sx, sh = W.nvfp4_scales(wl)
    dt, reps = 0.0, 0
    while (reps == 0 or dt < target_s) and reps < 1000:
        t0 = time.perf_counter()
        oracle.moe_layer_nvfp4(x, wr, W.host_bias(wl), bank_up, bank_down, sx, sh, wl.K, slot=slot)
        dt += time.perf_counter() - t0
        reps += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": reps * n_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_tokens} of the {wl.T} tokens of batch {seed_batch} ({wl.name}), full layer "
                      f"(router, top-{wl.K}, {len(used)} W4A4 experts in fp64 on dequantised codes, combine), "
                      f"{reps} times; {dt:.2f} s"}


def cpu_baseline_fp8_b128(wl, n_tokens, seed_batch=0, target_s=CPU_SAMPLE_SECONDS):
    """The oracle's W8A8 layer with FP8_B128 banks (router, experts, combine) on a token sample."""
    import numpy as np
    import oracle
    from synth import workloads as W
    x = W.host_x(wl, seed_batch)[:n_tokens]
    wr = W.host_router(wl)
    _, idx, _ = oracle.route(x, wr, W.host_bias(wl), wl.K)
    used = sorted(set(idx.reshape(-1).tolist()))
    slot = -np.ones(wl.E, dtype=np.int32)
    slot[used] = np.arange(len(used))
    key = (wl.name, 0, tuple(used), "fp8_b128")
    if key not in _BANKS:   # weight preparation: untimed
        _BANKS.clear()
        _BANKS[key] = (oracle.quantize_fp8_b128(W.host_w_up(wl, experts=used)),
                       oracle.quantize_fp8_b128(W.host_w_down(wl, experts=used)))
    bank_up, bank_down = _BANKS[key]
    sx, sh = W.fp8_b128_scales(wl)
    dt, reps = 0.0, 0
    while (reps == 0 or dt < target_s) and reps < 1000:
        t0 = time.perf_counter()
        oracle.moe_layer_fp8_b128(x, wr, W.host_bias(wl), bank_up, bank_down, sx, sh, wl.K, wl.H, wl.F, slot=slot)
        dt += time.perf_counter() - t0
        reps += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": reps * n_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_tokens} of the {wl.T} tokens of batch {seed_batch} ({wl.name}), FP8_B128 W8A8 layer "
                      f"(router, top-{wl.K}, {len(used)} experts in fp64, combine), {reps} times; {dt:.2f} s"}


def cpu_baseline_fp8(wl, n_tokens, seed_batch=0, layer=0, target_s=CPU_SAMPLE_SECONDS):
    """The oracle's W8A8 layer (norm, router, quantised experts, combine + residual) on a token sample."""
    import numpy as np
    import oracle
    import synth
    from synth import workloads as W
    x = synth.normal_bf16(synth.key(wl.seed, synth.T_X, seed_batch), n_tokens * wl.H, W.SIGMA_X).reshape(
        n_tokens, wl.H)
    wr = W.host_router(wl, layer)
    sx, sh = W.chain_scales()[layer]
    u = oracle.rmsnorm_bf16(x)
    _, idx, _ = oracle.route(u, wr, None, wl.K)
    used = sorted(set(idx.reshape(-1).tolist()))
    slot = -np.ones(wl.E, dtype=np.int32)
    slot[used] = np.arange(len(used))
    (qu, su), (qd, sd) = _host_banks(wl, layer, used, True)   # weight preparation: untimed
    dt, reps = 0.0, 0
    while (reps == 0 or dt < target_s) and reps < 1000:
        t0 = time.perf_counter()
        u = oracle.rmsnorm_bf16(x)
        oracle.moe_layer_fp8(u, wr, None, qu, su, qd, sd, sx, sh, wl.K, slot=slot, residual=x)
        dt += time.perf_counter() - t0
        reps += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": reps * n_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_tokens} tokens through layer {layer} of {wl.name} (norm, router, {len(used)} W8A8 "
                      f"experts in fp64 on dequantised codes, combine + residual), {reps} times; {dt:.2f} s"}


def run_native(args):
    import torch
    import torch.distributed as dist
    from synth import workloads as W

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
        barrier = lambda: dist.barrier()
    else:
        barrier = lambda: None
    device = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_kind = load_peaks()
    if args.gemm == "pair":
        import routed_expert_moe_b200 as moe
        moe.debug_set(3, 1)
    if args.pdl == "off":
        import routed_expert_moe_b200 as moe
        moe.debug_set(6, 0)

    wl = W.WORKLOADS[WORKLOADS[args.workload]]
    if wl.fp8 or wl.fp8_b128:
        f8 = probe_fp8_peak(device)
        if f8:
            peaks = dict(peaks, fp8_tflops=f8,
                         fp8_source="measured in this run: torch._scaled_mm e4m3 8192^3, best of 10 (burst)")
    layer = Chain(wl, device) if wl.layers > 1 else Layer(wl, device)
    launches = layer.launches_per_step()
    touched, rows = layer.touched_experts(0)
    import routed_expert_moe_b200 as _moe
    one_launch = ffn_is_one_launch(_moe, layer.dims if hasattr(layer, "dims") else layer.stack.dims)
    stages = stage_view(stage_profile(layer, max(3, min(args.steps, 20)), args.warmup), one_launch)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    ms = timed_loop(layer, args.steps, args.warmup, barrier)
    sampler.window(*timed_loop.window)
    clocks = sampler.stop()

    ms = reduce_max(ms, dist if ws > 1 else None, device)
    e2e_ms, bi, bo = e2e_loop(layer, args.steps, args.warmup)
    e2e_ms = reduce_max(e2e_ms, dist if ws > 1 else None, device)

    secondary = {}
    if not args.no_secondary and args.workload == "decode" and ws == 1:
        del layer
        torch.cuda.empty_cache()
        # the prefill chunk and the skewed (Zipf-routed) batch, each timed like the main line
        for key, name in (("secondary", "prefill"), ("secondary_skewed", "skewed")):
            wl2 = W.WORKLOADS[WORKLOADS[name]]
            layer2 = Layer(wl2, device, n_batches=2)
            t2, _ = layer2.touched_experts(0)
            st2 = stage_view(stage_profile(layer2, 10, 3), ffn_is_one_launch(_moe, layer2.dims))
            ms2 = timed_loop(layer2, 10, 3, barrier)
            secondary[key] = {"workload": wl2.name, "T": wl2.T, "tokens_per_s": wl2.T * 10 / (ms2 * 1e-3),
                              "ms_per_step": ms2 / 10, "touched_experts": t2, "stages_ms": st2,
                              "roofline": roofline_entry(wl2, st2, t2, peaks, peak_kind, name)}
            del layer2
            torch.cuda.empty_cache()

    if rank == 0:
        # MoE-layer tokens: a step of the chain passes T tokens through every layer
        value = job_value(ws, wl.T * wl.layers, args.steps, ms)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("fp8_e4m3 (W8A8) experts, bf16 router" if wl.fp8 else
                      "fp8_e4m3 FP8_B128 (W8A8, one fp32 weight scale per 128 along K) experts, bf16 router"
                      if wl.fp8_b128 else
                      "nvfp4 (W4A4: e2m1 codes, e4m3 block scales; fp16 tensor-core products) experts, bf16 router"
                      if wl.nvfp4 else "bf16"),
            "data": "synthetic: seeded N(0,1) activations, N(0,0.02) router/expert weights (bf16)",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "K": wl.K, "F": wl.F,
                       "layers": wl.layers, "touched_experts": touched, "shared_expert_width": wl.shared,
                       "l2": "inputs larger than L2: the touched experts' weights "
                             f"({(touched * wl.F + wl.shared) * wl.H * (1.125 if wl.nvfp4 else 2 if (wl.fp8 or wl.fp8_b128) else 4) * wl.layers / 1e9:.2f} GB) "
                             "stream from HBM every step; token batches rotate; no flush",
                       "parallelism": f"dp{ws} (independent token batches per GPU, weights replicated)",
                       "grouped_gemm": "cta_pair" if args.gemm == "pair" else "single_cta",
                       "programmatic_dependent_launch": args.pdl == "on"},
            "roofline": roofline_entry(wl, stages, touched, peaks, peak_kind, args.workload),
            "stages_ms": stages,
            "e2e": {"value": job_value(ws, wl.T * wl.layers, args.steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo},
            "gpu_launches": launches * args.steps,
            "clocks": clocks,
        }
        line.update(secondary)
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, 4 if wl.fp8 else 8 if (wl.nvfp4 or wl.fp8_b128) else min(wl.T, 64))
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


# --------------------------------------------------------------------------- expert parallelism

class EpLayer:
    """The layer split by expert over the ranks (routed_expert_moe_b200.ep): rank p owns experts
    [p*E/N, (p+1)*E/N) and routes its own batch; rows cross ranks in two all-to-alls."""

    def __init__(self, wl, device, n_batches=4):
        import torch
        import torch.distributed as dist
        import synth
        from routed_expert_moe_b200.ep import ExpertParallelLayer
        from synth import workloads as W
        self.wl, self.device = wl, device
        rank = dist.get_rank() if dist.is_initialized() else 0
        bf = torch.bfloat16
        stream = torch.cuda.current_stream().cuda_stream
        self.layer = ExpertParallelLayer(wl.H, wl.E, wl.K, wl.F) if dist.is_initialized() else None
        E_loc = self.layer.E_loc if self.layer else wl.E
        lo = rank * E_loc
        banks = []
        for tid, shape in ((synth.T_WUP, (wl.E, wl.F, wl.H)), (synth.T_WDOWN, (wl.E, wl.H, wl.F))):
            full = torch.empty(*shape, dtype=bf, device=device)
            synth.normal_bf16_device(synth.key(wl.seed, tid, 0), full.numel(), W.SIGMA_W, full.data_ptr(), stream)
            banks.append(full[lo:lo + E_loc].clone())
            del full
        self.wu, self.wd = banks
        self.wr = torch.empty(wl.E, wl.H, dtype=bf, device=device)
        synth.normal_bf16_device(synth.key(wl.seed, synth.T_WR, 0), self.wr.numel(), W.SIGMA_W, self.wr.data_ptr(),
                                 stream)
        self.xs = []
        for i in range(n_batches):   # each rank its own token batches
            x = torch.empty(wl.T, wl.H, dtype=bf, device=device)
            synth.normal_bf16_device(synth.key(wl.seed, synth.T_X, 16 * rank + i), x.numel(), W.SIGMA_X,
                                     x.data_ptr(), stream)
            self.xs.append(x)
        self.out = torch.empty(wl.T, wl.H, dtype=bf, device=device)
        torch.cuda.synchronize(device)

    def step(self, i, x=None, out=None):
        self.layer.forward(self.xs[i % len(self.xs)] if x is None else x, self.wr, None, self.wu, self.wd,
                           self.out if out is None else out)


# kernels of one expert-parallel pass beyond those of moe_forward: the regrouping, the owner's
# tile schedule, and the gather that returns the outputs in arrival order
EP_EXTRA_LAUNCHES = 3


def ep_line(ws, wl, steps, warmup, ms, e2e_ms, clocks, launches_per_step):
    """The JSON line of the expert-parallel mode: every rank processed wl.T tokens per step;
    ms and e2e_ms are the max over ranks."""
    nb = wl.T * wl.H * 2
    return {"metric": METRIC, "value": job_value(ws, wl.T, steps, ms), "unit": UNIT, "n_gpus": ws, "steps": steps,
            "warmup": warmup, "ms_per_step": ms / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) activations, N(0,0.02) router/expert weights (bf16)",
            "config": {"workload": wl.name, "T_per_rank": wl.T, "H": wl.H, "E": wl.E, "K": wl.K, "F": wl.F,
                       "parallelism": f"ep{ws} ({wl.E // ws} experts per rank, two NCCL all-to-alls per pass)",
                       "l2": "inputs larger than L2: each rank's experts stream from HBM every step"},
            "e2e": {"value": job_value(ws, wl.T, steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": nb, "d2h_bytes_per_step": nb},
            "gpu_launches": launches_per_step * steps, "clocks": clocks}


def run_ep(args):
    """--ep: the expert-parallel split under torchrun (one rank per GPU, NCCL)."""
    import datetime
    import torch
    import torch.distributed as dist
    from synth import workloads as W

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    if "MASTER_ADDR" not in os.environ:      # a single process without torchrun
        import socket
        so = socket.socket()
        so.bind(("127.0.0.1", 0))
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(so.getsockname()[1]), RANK="0", WORLD_SIZE="1")
        so.close()
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    barrier = lambda: dist.barrier()
    wl = W.WORKLOADS[WORKLOADS[args.workload]]
    layer = EpLayer(wl, device)
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    ms = timed_loop(layer, args.steps, args.warmup, barrier)
    sampler.window(*timed_loop.window)
    clocks = sampler.stop()
    ms = reduce_max(ms, dist, device)
    # end to end: this rank's batch from pinned host memory, its output back, every step
    hx = layer.xs[0].cpu().pin_memory()
    hout = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, pin_memory=True)
    dx = torch.empty_like(layer.xs[0])
    for i in range(args.warmup):
        dx.copy_(hx, non_blocking=True)
        layer.step(i, x=dx)
        hout.copy_(layer.out, non_blocking=True)
    barrier()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for i in range(args.steps):
        dx.copy_(hx, non_blocking=True)
        layer.step(i, x=dx)
        hout.copy_(layer.out, non_blocking=True)
    s1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(s0.elapsed_time(s1), dist, device)
    if rank == 0:
        import routed_expert_moe_b200 as moe
        launches = moe.forward_launches(moe.dims(wl.T, wl.H, wl.E, wl.K, wl.F)) + EP_EXTRA_LAUNCHES
        print(json.dumps(ep_line(ws, wl, args.steps, args.warmup, ms, e2e_ms, clocks, launches)), flush=True)
    dist.destroy_process_group()


# --------------------------------------------------------------------------- reference arm

def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from synth import workloads as W
    wl = W.WORKLOADS[WORKLOADS[args.workload]]
    n = 4 if wl.fp8 else min(wl.T, 16)
    for _ in range(args.warmup):
        cpu_baseline(wl, min(n, 4), target_s=0.0)
    vals = []
    t0 = time.perf_counter()
    for i in range(args.steps):
        vals.append(cpu_baseline(wl, n, target_s=0.0))   # one pass of the sample per step
    wall = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * n / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded N(0,1) activations, N(0,0.02) router/expert weights (bf16)",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "K": wl.K, "F": wl.F,
                       "sample_tokens_per_step": n},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": wall}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm", choices=["single", "pair"], default="single",
                    help="grouped GEMM on single CTAs, or on CTA pairs for tiles of more than 64 tokens")
    ap.add_argument("--ep", action="store_true",
                    help="time the expert-parallel split (experts divided over the ranks) instead of replicas")
    ap.add_argument("--pdl", choices=["on", "off"], default="on",
                    help="programmatic dependent launch between the layer's kernels")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.ep:
        run_ep(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
