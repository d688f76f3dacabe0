#!/usr/bin/env python
"""Benchmark of the W4A8 per-channel linear layer on B200.

Default run: both halves of the metric on one JSON line.
  * decode (the line's value): the decode single linear, K = N = 4096,
    activation rows M in {1, 4, 16}. One step = one pass of the run-time hot
    path over one batch: for each M, w4a8_linear (dynamic INT8 quantization of
    X[M][4096], the W4A8 product, dequantization). HBM GB/s of algorithmic
    bytes (packed weights + weight scales + float32 X + float32 Y per linear)
    per second of device time. Weight buffers rotate through a pool of
    distinct copies several times larger than L2, so every launch streams its
    weights from HBM.
  * prefill (the "prefill" sub-record): M = 2048, K = 4096, N = 11008,
    float32 out; one step = one w4a8_linear (activation pass + tensor-core
    GEMM + epilogue); TOPS = 2 M N K per second, and the GEMM kernel alone
    against the dense INT8 tensor peak.
The weights are quantized and packed once, offline, before timing (their
quantize+pack pass is timed on its own and reported under "stages").

Timing: CUDA graphs of the timed steps are built and replayed untimed first
(warm-up), then the same graphs run the --steps-long region `repeats` times
back to back, each bracketed by CUDA events on the launching stream; the
reported time is the median region. Multi-GPU (torchrun): every rank runs the
same independent workload (weak scaling, no collective on the data path);
time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|...]
"""
from __future__ import annotations

import argparse
import concurrent.futures
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A8 linear: TOPS (prefill) and HBM GB/s (decode) vs B200 roofline"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernels, from ncu captures of this file's own workloads, stored
# with a hash of the kernel sources they were taken on: a figure whose hash no
# longer matches the sources is reported as null (stale).
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
KERNEL_SOURCES = (os.path.join(ROOT, "w4a8_quantized_gemm_channel_b200", "csrc"), os.path.join(ROOT, "include"))
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0   # nominal dense ratio (4.5 vs 2.25 PFLOP/s)
GRAPH_STEPS = 16
MIN_TIMED_S = 0.5      # repeat the timed region until this much device time is covered
MAX_REPEATS = 2000


def source_hash() -> str:
    """sha256 over the kernel sources (csrc/*.cu, *.cuh and include/*.h)."""
    h = hashlib.sha256()
    for d in KERNEL_SOURCES:
        for name in sorted(os.listdir(d)):
            if name.endswith((".cu", ".cuh", ".h")):
                h.update(name.encode())
                with open(os.path.join(d, name), "rb") as f:
                    h.update(f.read())
    return h.hexdigest()


def traffic_for(kernel: str, workload: str):
    """(bytes per launch, note) from the committed ncu figures, or (None, why)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None, "no ncu traffic figures committed"
    e = d.get("kernels", {}).get(f"{kernel}@{workload}")
    if e is None:
        return None, f"no ncu capture of {kernel} on this workload"
    if d.get("source_sha256") != source_hash():
        return None, f"stale: the kernel sources changed since the ncu capture of {kernel}"
    return e["dram_bytes_per_launch"], (f"dram__bytes_read.sum + dram__bytes_write.sum per {kernel} launch, "
                                        f"{e.get('launches', '?')} captured launches ({e.get('case', workload)})")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks ---

class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        self.summary = self._stop()
        return self.summary

    def _stop(self) -> dict:
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax or None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- workloads ---

class DecodeWorkload:
    """K = N = 4096, M in {1, 4, 16}; weights N(0, 0.02), X N(0, 1) with 8
    outlier channels x20."""
    name = "decode"

    def __init__(self, torch, native, synth, device, l2_bytes, w8=False, zp=False, grp=False):
        self.torch, self.nat = torch, native
        self.w8 = w8  # the W8A8 path: INT8 weight rows instead of packed INT4
        self.zpf = zp  # the zero-point INT4 path: asymmetric per-channel weights
        self.grp = grp  # the group-wise INT4 path: scale and zero point per 128 weights
        self.K, self.N, self.MS = synth.DECODE_K, synth.DECODE_N, synth.DECODE_MS
        w = synth.decode_case(1).w
        self.w_host = w
        wd = torch.from_numpy(w).to(device)
        if grp:
            wp, sw, zpt = native.w4g_quantize_pack(wd)
        elif zp:
            wp, sw, zpt = native.w4z_quantize_pack(wd)
        else:
            wp, sw = native.w8_quantize(wd) if w8 else native.w4_quantize_pack(wd)
        self.wd = wd
        per_weight = wp.numel() + 4 * sw.numel() * (2 if (zp or grp) else 1)
        # enough distinct copies (>= 3x L2) that each launch's weights were
        # evicted from L2 since their last use
        need = -(-3 * l2_bytes // per_weight) + len(self.MS)
        self.pool = -(-need // len(self.MS)) * len(self.MS)
        self.wp = [wp.clone() for _ in range(self.pool)]
        self.sw = [sw.clone() for _ in range(self.pool)]
        self.zp = [zpt.clone() for _ in range(self.pool)] if (zp or grp) else None
        self.x_host = {m: synth.decode_case(m).x for m in self.MS}
        self.x = {m: torch.from_numpy(self.x_host[m]).to(device) for m in self.MS}
        self.y = {m: torch.empty((m, self.N), dtype=torch.float32, device=device) for m in self.MS}
        ws_size = (lambda m: native.lib.w4z_workspace_size(m, self.K, self.N)) if zp else \
            (lambda m: native.workspace_size(m, self.K))
        self.ws = {m: torch.empty(ws_size(m), dtype=torch.uint8, device=device) for m in self.MS}
        self.slot = 0
        self.pool_bytes = self.pool * per_weight

    def weight_ld(self):
        return self.nat.w8a8_ld(self.K) if self.w8 else self.nat.packed_ld(self.K)

    def linear_q(self, xq, sx, k, wp, sw, **kw):
        if self.zpf or self.grp:
            i = next(j for j, t in enumerate(self.wp) if t is wp)
            if self.grp:
                return self.nat.w4g_linear_q(xq, sx, k, wp, sw, self.zp[i], **kw)
            return self.nat.w4z_linear_q(xq, sx, k, wp, sw, self.zp[i], workspace=self.ws[xq.shape[0]], **kw)
        return (self.nat.w8a8_linear_q if self.w8 else self.nat.w4a8_linear_q)(xq, sx, k, wp, sw, **kw)

    def bytes_per_step(self):
        ldp = self.weight_ld()
        # scales (and zero points) per launch: sw [N]; zero-point: + zp [N]; group-wise: sa, zp [N][ng]
        scales = 8 * self.N if self.zpf else (8 * self.sw[0].numel() if self.grp else 4 * self.N)
        return sum(self.N * ldp + scales + 4 * m * self.K + 4 * m * self.N for m in self.MS)

    def ops_per_step(self):
        return sum(2 * m * self.N * self.K for m in self.MS)

    def launches_per_step(self):
        """Kernels one step enqueues, as the library reports them."""
        n = 0
        for m in self.MS:
            self.call(m, 0)
            n += self.nat.last_launch_count()
        self.torch.cuda.synchronize()
        return n

    def call(self, m, s, x=None):
        # weights were quantized before timing and the stream has synchronized
        # since: the serving-style call promises they are settled
        xx = self.x[m] if x is None else x
        if self.grp:
            self.nat.w4g_linear(xx, self.wp[s], self.sw[s], self.zp[s], y=self.y[m], workspace=self.ws[m],
                                static_weights=True)
            return
        if self.zpf:
            self.nat.w4z_linear(xx, self.wp[s], self.sw[s], self.zp[s], y=self.y[m], workspace=self.ws[m],
                                static_weights=True)
            return
        lin = self.nat.w8a8_linear if self.w8 else self.nat.w4a8_linear
        lin(xx, self.wp[s], self.sw[s], y=self.y[m], workspace=self.ws[m], static_weights=True)

    def step(self):
        for m in self.MS:
            s = self.slot
            self.slot = (self.slot + 1) % self.pool
            self.call(m, s)

    def config(self):
        form = " W8A8" if self.w8 else (" zero-point INT4" if self.zpf else
                                        (" group-wise INT4 (128)" if self.grp else ""))
        return {"workload": f"decode single linear{form} K={self.K} N={self.N} "
                            f"M in {list(self.MS)}",
                "K": self.K, "N": self.N, "M": list(self.MS),
                "l2": f"inputs larger than L2: {self.pool} distinct packed weight buffers "
                      f"({self.pool_bytes / 1e6:.0f} MB) rotate across launches",
                "weights": "N(0,0.02) quantized" + ("" if self.w8 else "+packed") + " once before timing",
                "activations": "N(0,1), 8 input channels x20",
                "call": ("w8a8_linear" if self.w8 else "w4z_linear" if self.zpf else
                         "w4g_linear" if self.grp else "w4a8_linear")
                        + " with W4A8_STATIC_WEIGHTS"}


class PrefillWorkload:
    """M = 2048, K = 4096, N = 11008 (MLP up-projection shape); weights
    N(0, 0.02); X N(0, 1) with 0.5% of input channels x20. One step = one
    w4a8_linear (activation quantization + tensor-core GEMM + epilogue)."""
    name = "prefill"

    def __init__(self, torch, native, synth, device, l2_bytes, relu=False, w8=False, grp=False):
        self.torch, self.nat = torch, native
        self.w8 = w8
        self.grp = grp  # group-wise INT4 (scale and zero point per 128 weights)
        c = synth.prefill_case()
        self.M, self.K, self.N = c.x.shape[0], c.w.shape[0], c.w.shape[1]
        self.MS = (self.M,)
        self.relu = relu
        wd = torch.from_numpy(c.w).to(device)
        self.wd = wd
        self.zp = None
        if grp:
            wp, sw, self.zp = native.w4g_quantize_pack(wd)
        else:
            wp, sw = native.w8_quantize(wd) if w8 else native.w4_quantize_pack(wd)
        per_set = wp.numel() + 4 * self.M * self.K + 4 * self.M * self.N
        self.pool = max(2, -(-3 * l2_bytes // per_set))
        self.wp = [wp.clone() for _ in range(self.pool)]
        self.sw = [sw.clone() for _ in range(self.pool)]
        self.x_host = {self.M: c.x}
        x = torch.from_numpy(c.x).to(device)
        self.xs = [x.clone() for _ in range(self.pool)]
        self.x = {self.M: x}
        self.ys = [torch.empty((self.M, self.N), dtype=torch.float32, device=device) for _ in range(self.pool)]
        self.y = {self.M: self.ys[0]}
        self.ws = {self.M: torch.empty(native.workspace_size(self.M, self.K), dtype=torch.uint8, device=device)}
        self.slot = 0
        self.pool_bytes = self.pool * per_set

    def bytes_per_step(self):
        ldp = self.nat.w8a8_ld(self.K) if self.w8 else self.nat.packed_ld(self.K)
        return self.N * ldp + 4 * self.N + 4 * self.M * self.K + 4 * self.M * self.N

    def ops_per_step(self):
        return 2 * self.M * self.N * self.K

    def launches_per_step(self):
        """Kernels one step enqueues, as the library reports them."""
        self.step()
        n = self.nat.last_launch_count()
        self.torch.cuda.synchronize()
        return n

    def step(self):
        s = self.slot
        self.slot = (self.slot + 1) % self.pool
        if self.grp:
            self.nat.w4g_linear(self.xs[s], self.wp[s], self.sw[s], self.zp, relu=self.relu, y=self.ys[s],
                                workspace=self.ws[self.M])
            return
        lin = self.nat.w8a8_linear if self.w8 else self.nat.w4a8_linear
        lin(self.xs[s], self.wp[s], self.sw[s], relu=self.relu, y=self.ys[s], workspace=self.ws[self.M])

    def config(self):
        form = " W8A8" if self.w8 else (" group-wise INT4 (128)" if self.grp else "")
        return {"workload": f"prefill single linear{form} M={self.M} K={self.K} "
                            f"N={self.N}" + (" +ReLU" if self.relu else ""),
                "M": self.M, "K": self.K, "N": self.N,
                "l2": f"inputs larger than L2: {self.pool} distinct X/W/Y sets "
                      f"({self.pool_bytes / 1e6:.0f} MB) rotate across launches"}


# ------------------------------------------------------------ timing core ---

def max_over_ranks(torch, dist, value: float, device) -> float:
    """The slowest rank's time (every rank gets it); identity on one rank."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def build_graphs(torch, wl, nsteps):
    """CUDA graphs that run exactly nsteps steps: `full` replays of one
    GRAPH_STEPS-step graph, then one graph of the remainder."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):           # warm the library's per-device state outside capture
            wl.step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    full, rem = divmod(nsteps, GRAPH_STEPS)
    g = None
    if full:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(GRAPH_STEPS):
                wl.step()
    gr = None
    if rem:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for _ in range(rem):
                wl.step()
    return g, full, gr


PREROLL_S = 0.3         # untimed load before a sampled region, so every clock sample is under load


def timed_repeats(torch, enqueue, dist=None, device=None, min_repeats=5, min_s=None, clocks=None):
    """Median device time (ms) of one `enqueue()` (already warmed) over
    back-to-back repeats, each bracketed by CUDA events on the current stream;
    repeats run until min_s (default MIN_TIMED_S) of device time is covered
    (at least min_repeats, at most MAX_REPEATS; the same count on every
    rank). With `clocks`, the sampler starts before an untimed pre-roll of
    PREROLL_S and stops right after the timed repeats. Returns (median ms,
    repeats)."""
    min_s = MIN_TIMED_S if min_s is None else min_s
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    enqueue()
    b.record()
    torch.cuda.synchronize()
    one = max(a.elapsed_time(b), 1e-3)
    reps = int(min(MAX_REPEATS, max(min_repeats, -(-min_s * 1e3 // one))))
    reps = int(max_over_ranks(torch, dist, float(reps), device))
    if clocks is not None:
        clocks.start()
        for _ in range(int(min(MAX_REPEATS, max(1, min(PREROLL_S, min_s) * 1e3 // one)))):
            enqueue()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    evs[0].record()
    for i in range(reps):
        enqueue()
        evs[i + 1].record()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.stop()
    if dist is not None:
        dist.barrier()
    return statistics.median(evs[i].elapsed_time(evs[i + 1]) for i in range(reps)), reps


def time_steps(torch, wl, steps, warmup, dist=None, device=None, clocks=None):
    """Median device time (ms) of a region of exactly `steps` steps, and the
    repeat count. The timed graphs themselves run the warm-up (at least
    `warmup` steps, and every graph at least once), so no graph is replayed
    for the first time inside a timed region."""
    g, full, gr = build_graphs(torch, wl, steps)

    def region():
        for _ in range(full):
            g.replay()
        if gr is not None:
            gr.replay()
    for _ in range(max(1, -(-warmup // steps))):
        region()
    torch.cuda.synchronize()
    return timed_repeats(torch, region, dist, device, clocks=clocks)


def _graph_of(torch, run):
    """Capture run() (after one eager warm-up on a side stream) and replay it
    three times untimed."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    return g


def time_kernel_only(torch, nat, wl):
    """Device time per decode-kernel launch (w4a8_linear_q, INT8 activations
    already quantized) in a back-to-back graph over the rotating weight pool,
    per M (median over repeats of the graph); returns {m: (ms_per_launch,
    algorithmic_bytes, kernel_name)}."""
    out = {}
    ldp = wl.weight_ld()
    for m in wl.MS:
        xq, sx = nat.a8_quantize_rows(wl.x[m])
        reps = wl.pool

        def run():
            for i in range(reps):
                wl.linear_q(xq, sx, wl.K, wl.wp[i], wl.sw[i], y=wl.y[m], static_weights=True)
        wl.linear_q(xq, sx, wl.K, wl.wp[0], wl.sw[0], y=wl.y[m], static_weights=True)
        kernel = nat.last_kernel()
        g = _graph_of(torch, run)
        ms, _ = timed_repeats(torch, g.replay, min_repeats=20)
        ms /= reps
        nbytes = wl.N * ldp + 4 * wl.N + m * xq.shape[1] + 4 * m + 4 * m * wl.N
        if getattr(wl, "zpf", False):
            nbytes += 4 * wl.N  # the zero points
        if getattr(wl, "grp", False):
            nbytes += 8 * wl.sw[0].numel() - 4 * wl.N  # per-group scales and zero points
        out[m] = (ms, nbytes, kernel)
    return out


def time_gemm_only(torch, nat, wl):
    """Device time per tensor-core GEMM launch (w4a8_linear_q on INT8
    activations, the kernel the library picks for the shape) over the
    rotating buffer sets (median over repeats)."""
    xqs = [nat.a8_quantize_rows(x) for x in wl.xs]
    lin_q = nat.w8a8_linear_q if wl.w8 else nat.w4a8_linear_q

    def run():
        for i in range(wl.pool):
            xq, sx = xqs[i]
            if wl.grp:
                nat.w4g_linear_q(xq, sx, wl.K, wl.wp[i], wl.sw[i], wl.zp, relu=wl.relu, y=wl.ys[i], path="tc")
            else:
                lin_q(xq, sx, wl.K, wl.wp[i], wl.sw[i], relu=wl.relu, y=wl.ys[i])
    g = _graph_of(torch, run)
    # a kernel timed alone: a short burst after the device had a moment to
    # leave the power cap the long step region may have reached
    time.sleep(1.0)
    ms, _ = timed_repeats(torch, g.replay, min_repeats=10, min_s=0.0)
    return ms / wl.pool


def time_quantize_pack(torch, nat, wl):
    """The offline weight pass (steps 1-2) on the decode weight matrix."""
    wp, sw = nat.w4_quantize_pack(wl.wd)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 20
    start.record()
    for _ in range(reps):
        nat.w4_quantize_pack(wl.wd, wp=wp, sw=sw)
    stop.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop) / reps
    nbytes = wl.wd.numel() * 4 + wp.numel() + 4 * sw.numel()
    return ms, nbytes


def time_e2e(torch, nat, wl, steps):
    """Same metric through the public call with host buffers: every step
    copies X from pinned host memory and reads Y back."""
    xh = {m: torch.from_numpy(wl.x_host[m]).pin_memory() for m in wl.MS}
    yh = {m: torch.empty((m, wl.N), dtype=torch.float32).pin_memory() for m in wl.MS}
    xd = {m: torch.empty_like(wl.x[m]) for m in wl.MS}

    def one(slot):
        for j, m in enumerate(wl.MS):
            s = (slot * len(wl.MS) + j) % wl.pool
            xd[m].copy_(xh[m], non_blocking=True)
            wl.call(m, s, x=xd[m])
            yh[m].copy_(wl.y[m], non_blocking=True)
    for i in range(5):
        one(i)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        one(i)
    stop.record()
    torch.cuda.synchronize()
    h2d = sum(xh[m].numel() * 4 for m in wl.MS)
    d2h = sum(yh[m].numel() * 4 for m in wl.MS)
    return start.elapsed_time(stop), h2d, d2h


def time_e2e_prefill(torch, nat, wl, steps):
    """The prefill step through w4a8_linear with host buffers: X copied in
    from pinned memory and Y read back every step."""
    xh = torch.from_numpy(wl.x_host[wl.M]).pin_memory()
    yh = torch.empty((wl.M, wl.N), dtype=torch.float32).pin_memory()
    xd = torch.empty_like(wl.xs[0])

    def one(slot):
        s = slot % wl.pool
        xd.copy_(xh, non_blocking=True)
        nat.w4a8_linear(xd, wl.wp[s], wl.sw[s], relu=wl.relu, y=wl.ys[s], workspace=wl.ws[wl.M])
        yh.copy_(wl.ys[s], non_blocking=True)
    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        one(i)
    stop.record()
    torch.cuda.synchronize()
    return start.elapsed_time(stop), xh.numel() * 4, yh.numel() * 4


# ------------------------------------------------------- the CPU oracle ---

def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_columns(pool, oracle, xq, sx, wp, sw, k, c0, c1, per):
    """oracle.linear_q on output channels [c0, c1) in tasks of `per` channels
    spread over the thread pool (the oracle's C calls release the GIL)."""
    jobs = [pool.submit(oracle.linear_q, xq, sx, wp[a:min(a + per, c1)], sw[a:min(a + per, c1)], k)
            for a in range(c0, c1, per)]
    return [j.result() for j in jobs]


def oracle_decode_steps(budget_s: float, threads: int, min_steps: int = 1, max_steps: int | None = None):
    """The oracle as it stands, timed on the decode workload at full size
    (K = N = 4096, M = 1, 4, 16; per M the activation pass, then the product
    and dequantization over all output channels split across `threads`
    threads) until `budget_s` seconds are spent. Returns (GB/s of the decode
    line's algorithmic bytes, seconds, steps)."""
    import oracle
    from w4a8_quantized_gemm_channel_b200 import synth
    k, n = synth.DECODE_K, synth.DECODE_N
    wp, sw = oracle.w4_quantize_pack(synth.decode_case(1).w)   # offline step, not timed
    xs = {m: synth.decode_case(m).x for m in synth.DECODE_MS}
    ldp = wp.shape[1]
    step_bytes = sum(n * ldp + 4 * n + 4 * m * k + 4 * m * n for m in xs)
    per = max(8, n // (4 * threads))
    steps = 0
    with concurrent.futures.ThreadPoolExecutor(threads) as pool:
        t0 = time.perf_counter()
        while (time.perf_counter() - t0 < budget_s or steps < min_steps) and (max_steps is None or steps < max_steps):
            for m, x in xs.items():
                xq, sx = oracle.a8_quantize_rows(x)
                _oracle_columns(pool, oracle, xq, sx, wp, sw, k, 0, n, per)
            steps += 1
        t = time.perf_counter() - t0
    return steps * step_bytes / t / 1e9, t, steps


def oracle_prefill_rate(budget_s: float, threads: int, case):
    """The oracle on the prefill workload (M = 2048, K = 4096, N = 11008):
    the activation pass over all of X, then the product on as many output
    channels as `budget_s` seconds allow (full M and K, split across
    `threads` threads). The full-layer time is extrapolated from that sample:
    t = t_activation + t_sample * N / channels_done. Returns (TOPS, detail)."""
    import oracle
    x, w = case.x, case.w
    m, k = x.shape
    n = w.shape[1]
    wp, sw = oracle.w4_quantize_pack(w)   # offline step, not timed
    t0 = time.perf_counter()
    xq, sx = oracle.a8_quantize_rows(x)
    t_q = time.perf_counter() - t0
    per, done, t_p = 4, 0, 0.0
    with concurrent.futures.ThreadPoolExecutor(threads) as pool:
        while done < n and (t_p < budget_s or done == 0):
            c1 = min(n, done + per * threads)
            t1 = time.perf_counter()
            _oracle_columns(pool, oracle, xq, sx, wp, sw, k, done, c1, per)
            t_p += time.perf_counter() - t1
            done = c1
    t_full = t_q + t_p * n / done
    return 2.0 * m * n * k / t_full / 1e12, {"channels": done, "t_act_s": round(t_q, 3), "t_sample_s": round(t_p, 3)}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle on the decode line's workload, on the
    host cores, W untimed and K timed steps (each a full decode step, or a
    bounded sample of one if the budget is too small for full steps)."""
    if rank != 0:
        return
    threads = cpu_threads()
    oracle_decode_steps(0.0, threads, min_steps=max(1, min(args.warmup, 3)), max_steps=max(1, min(args.warmup, 3)))
    gbs, t, steps = oracle_decode_steps(args.cpu_budget, threads, min_steps=args.steps, max_steps=args.steps)
    sample = f"{steps} full decode steps (M = 1, 4, 16; K = N = 4096) on {threads} threads, {t:.2f} s"
    line = {"metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "impl": "reference",
            "ms_per_step": round(t * 1e3 / steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "decode single linear K=4096 N=4096 M in [1, 4, 16]",
                       "note": "CPU oracle (plain C, one call per output-channel chunk, thread pool)"},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def prefill_record(args, torch, native, synth, device, props, dist, world, rank, relu=False, w8=False,
                   cpu=None, grp=False):
    """Time the prefill workload: the step (w4a8_linear, activation pass
    included), the tensor-core GEMM alone, and the step through host buffers.
    Returns the record (value in TOPS, with roofline, clocks and launches)."""
    wl = PrefillWorkload(torch, native, synth, device, props.L2_cache_size, relu=relu, w8=w8, grp=grp)
    clocks = ClockSampler(device.index or 0)
    ms, repeats = time_steps(torch, wl, args.steps, args.warmup, dist, device, clocks=clocks)
    ck = clocks.summary
    ms = max_over_ranks(torch, dist, ms, device)
    tops = world * args.steps * wl.ops_per_step() / (ms * 1e-3) / 1e12
    g_ms = time_gemm_only(torch, native, wl)
    peaks, kind = measured_peaks()
    peak = INT8_OVER_BF16 * float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    achieved = wl.ops_per_step() / (g_ms * 1e-3) / 1e12
    kname = native.last_kernel()  # the product kernel the library picked for this shape
    traffic, tnote = traffic_for(kname, "prefill" + ("-w8a8" if w8 else "") + ("-grp" if grp else "")
                                 + ("-relu" if relu else ""))
    e2e_steps = min(args.steps, 10)
    e_ms, h2d, d2h = time_e2e_prefill(torch, native, wl, e2e_steps) if not (w8 or grp) else (None, 0, 0)
    rec = {"value": round(tops, 2), "unit": "TOPS", "steps": args.steps, "repeats": repeats,
           "ms_per_step": round(ms / args.steps, 6),
           "dtype": "s8xs8->s32" if w8 else ("s8xu4(group zp)->f32" if grp else "s8xs4->s32"),
           "config": wl.config(),
           "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                        "unit": "TOPS", "frac": round(achieved / peak, 4),
                        "peak_source": f"{kind} bf16_tflops (burst) x {INT8_OVER_BF16:g}, the nominal dense "
                                       "int8/bf16 ratio (4.5 / 2.25 PFLOP/s); the kernel is timed alone, in a "
                                       "burst of back-to-back launches",
                        "peak_sustained": round(INT8_OVER_BF16 * float(peaks.get("bf16_tflops_sustained", 1400.0)), 1),
                        "traffic": traffic, "traffic_note": tnote,
                        "kernel": kname + " (" + ("w8a8" if w8 else ("w4g" if grp else "w4a8"))
                                  + "_linear_q back to back over rotating buffers)", "us": round(g_ms * 1e3, 2)},
           "gpu_launches": args.steps * wl.launches_per_step(), "clocks": ck}
    if e_ms is not None:
        rec["e2e"] = {"value": round(world * e2e_steps * wl.ops_per_step() / (e_ms * 1e-3) / 1e12, 2),
                      "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}
    if cpu is not None:
        rec["cpu_baseline"] = cpu
    del wl
    torch.cuda.empty_cache()
    return rec


def run_prefill(args, torch, native, synth, device, props, dist, world, rank, relu=False, w8=False, cpu=None,
                grp=False):
    rec = prefill_record(args, torch, native, synth, device, props, dist, world, rank, relu=relu, w8=w8, cpu=cpu,
                         grp=grp)
    line = {"metric": METRIC, "value": rec.pop("value"), "unit": rec.pop("unit"), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": rec.pop("dtype"),
            "data": "synthetic", **rec}
    if rank == 0:
        print(json.dumps(line), flush=True)


def decode_record(args, torch, native, synth, device, props, dist, world, form="w4"):
    """Time the decode workload in one weight form ("w4": W4A8; "w8": W8A8;
    "zp": zero-point INT4; "grp": group-wise INT4): the step (the form's
    linear call at M = 1, 4, 16, activation quantization included), the
    product call alone per M, the step through host buffers (W4A8) and the
    offline weight pass (W4A8). Returns the line's fields."""
    wl = DecodeWorkload(torch, native, synth, device, props.L2_cache_size, w8=form == "w8", zp=form == "zp",
                        grp=form == "grp")
    clocks = ClockSampler(device.index or 0)
    ms, repeats = time_steps(torch, wl, args.steps, args.warmup, dist, device, clocks=clocks)
    ck = clocks.summary
    ms = max_over_ranks(torch, dist, ms, device)
    bytes_step = wl.bytes_per_step()
    value = world * args.steps * bytes_step / (ms * 1e-3) / 1e9

    kern = time_kernel_only(torch, native, wl)
    # the dominant product kernel: the one with the most device time over the step's M
    by_kernel = {}
    for m, (_, _, name) in kern.items():
        by_kernel.setdefault(name, []).append(m)
    dom = max(by_kernel, key=lambda name: sum(kern[m][0] for m in by_kernel[name]))
    dom_ms = by_kernel[dom]
    k_ms = sum(kern[m][0] for m in dom_ms)
    k_bytes = sum(kern[m][1] for m in dom_ms)
    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    achieved = k_bytes / (k_ms * 1e-3) / 1e9
    wname = {"w4": "decode", "w8": "decode-w8a8", "zp": "decode-zp", "grp": "decode-grp"}[form]
    traffic, tnote = traffic_for(dom, wname)
    call = {"w4": "w4a8_linear_q", "w8": "w8a8_linear_q", "zp": "w4z_linear_q", "grp": "w4g_linear_q"}[form]
    rec = {
        "value": round(value, 2), "unit": "GB/s", "steps": args.steps, "repeats": repeats,
        "ms_per_step": round(ms / args.steps, 6),
        "dtype": {"w4": "s8xs4->s32", "w8": "s8xs8->s32", "zp": "s8xu4(zp)->s32", "grp": "s8xu4(group zp)->f32"}[form],
        "config": wl.config(),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                     "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "peak_source": f"{peak_kind} hbm_gbs", "traffic": traffic, "traffic_note": tnote,
                     "kernel": f"{dom} over M in {dom_ms} ({call} back to back over rotating "
                               "weights, static-weights promise); per_m lists every M's kernel",
                     "per_m": {str(m): {"kernel": v[2], "us": round(v[0] * 1e3, 3), "bytes": v[1],
                                        "gbs": round(v[1] / (v[0] * 1e-3) / 1e9, 1)}
                               for m, v in kern.items()}},
        "tops": round(world * args.steps * wl.ops_per_step() / (ms * 1e-3) / 1e12, 4),
        "gpu_launches": args.steps * wl.launches_per_step(),
        "gpu_launches_note": "kernels per timed region of `steps` steps (the region ran `repeats` times)",
        "clocks": ck,
    }
    if form == "w4":
        qp_ms, qp_bytes = time_quantize_pack(torch, native, wl)
        rec["stages"] = {"quantize_pack": {"ms": round(qp_ms, 4), "bytes": qp_bytes,
                                           "gbs": round(qp_bytes / (qp_ms * 1e-3) / 1e9, 1),
                                           "frac_hbm": round(qp_bytes / (qp_ms * 1e-3) / 1e9 / hbm_peak, 4),
                                           "shape": f"K={wl.K} N={wl.N} fp32 -> packed"}}
        e2e_steps = min(args.steps, 2000)
        e2e_ms, h2d, d2h = time_e2e(torch, native, wl, e2e_steps)
        rec["e2e"] = {"value": round(world * e2e_steps * bytes_step / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}
    del wl
    torch.cuda.empty_cache()
    return rec


def run_decode_w8a8(args, torch, native, synth, device, props, dist, world, rank, zp=False, grp=False):
    """The decode workload on the W8A8 path (or the zero-point / group-wise
    INT4 paths): one JSON line."""
    rec = decode_record(args, torch, native, synth, device, props, dist, world,
                        form="zp" if zp else ("grp" if grp else "w8"))
    line = {"metric": METRIC, "value": rec.pop("value"), "unit": rec.pop("unit"), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": rec.pop("dtype"),
            "data": "synthetic", **rec}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_sweep(torch, native, synth, device, props):
    """Kernel time per shape of the Gemma3-1B stack and the 70B-shaped layers
    (w4a8_linear end to end on device-resident inputs, back-to-back in a
    graph over rotating weight copies)."""
    peaks, _ = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    tc = INT8_OVER_BF16 * float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    shapes = [("gemma_" + nm, k, n, m, 0.02) for (nm, k, n) in synth.GEMMA_PROJ for m in synth.GEMMA_MS]
    shapes += [(f"llama70_{k}x{n}", k, n, m, 0.01) for (k, n) in synth.LLAMA70_SHAPES for m in synth.LLAMA70_MS]
    for name, k, n, m, std in shapes:
        w = torch.from_numpy(synth.linear_weights(k, n, std, seed=3)).to(device)
        wp, sw = native.w4_quantize_pack(w)
        del w
        x = torch.from_numpy(synth.linear_activations(m, k, seed=3)[0]).to(device)
        per = wp.numel() + 4 * m * k + 4 * m * n
        pool = max(2, min(64, -(-3 * props.L2_cache_size // per)))
        wps = [wp.clone() for _ in range(pool)]
        sws = [sw.clone() for _ in range(pool)]
        y = torch.empty((m, n), dtype=torch.float32, device=device)
        ws = torch.empty(native.workspace_size(m, k), dtype=torch.uint8, device=device)

        def run():
            for i in range(pool):
                native.w4a8_linear(x, wps[i], sws[i], y=y, workspace=ws)
        run()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        g.replay()
        torch.cuda.synchronize()
        reps = max(3, int(2e9 // max(1, 2 * m * n * k * pool)))
        reps = min(reps, 200)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(reps):
            g.replay()
        stop.record()
        torch.cuda.synchronize()
        us = start.elapsed_time(stop) * 1e3 / (reps * pool)
        nbytes = n * native.packed_ld(k) + 4 * n + 4 * m * k + 4 * m * n
        ops = 2 * m * n * k
        gbs = nbytes / (us * 1e-6) / 1e9
        tops = ops / (us * 1e-6) / 1e12
        frac = max(gbs / hbm, tops / tc)
        print(json.dumps({"shape": name, "M": m, "K": k, "N": n, "us": round(us, 3),
                          "GBs": round(gbs, 1), "TOPS": round(tops, 2), "roofline_frac": round(frac, 4),
                          "path": native.last_path(), "kernel": native.last_kernel()}), flush=True)
        del wps, sws, wp, sw, x, y, ws, g
        torch.cuda.empty_cache()


def run_gemma_stack(torch, native, synth, device, steps=20):
    """The Gemma3-1B-shaped stack: 26 layers x 7 projections = 182 independent
    linears (distinct quantized weights, 349 MB packed), run back to back in
    one CUDA graph per M, with the static-weights promise. One JSON line per
    M with the aggregate and per-projection-type rates; the roofline fraction
    is max(T_mem, T_tc) / T_measured over the algorithmic bytes and ops."""
    peaks, _ = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    tc = INT8_OVER_BF16 * float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    layers = []
    for layer in range(synth.GEMMA_LAYERS):
        row = []
        for p in range(len(synth.GEMMA_PROJ)):
            w = torch.from_numpy(synth.gemma_weights(layer, p)).to(device)
            row.append(native.w4_quantize_pack(w))
            del w
        layers.append(row)
    torch.cuda.synchronize()

    def timed_graph(calls):
        for c in calls:
            c()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in calls:
                c()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            g.replay()
        stop.record()
        torch.cuda.synchronize()
        return start.elapsed_time(stop) * 1e3 / steps  # us per replay

    for m in synth.GEMMA_MS:
        xs = [torch.from_numpy(synth.gemma_activations(m, k, sub=p)).to(device)
              for p, (_, k, _) in enumerate(synth.GEMMA_PROJ)]
        ys = [torch.empty((m, n), dtype=torch.float32, device=device) for (_, _, n) in synth.GEMMA_PROJ]
        wss = [torch.empty(native.workspace_size(m, k), dtype=torch.uint8, device=device)
               for (_, k, _) in synth.GEMMA_PROJ]

        def call(layer, p):
            wp, sw = layers[layer][p]
            return lambda: native.w4a8_linear(xs[p], wp, sw, y=ys[p], workspace=wss[p], static_weights=True)

        def work(ps):
            nbytes = ops = 0
            for p in ps:
                _, k, n = synth.GEMMA_PROJ[p]
                nbytes += synth.GEMMA_LAYERS * (n * native.packed_ld(k) + 4 * n + 4 * m * k + 4 * m * n)
                ops += synth.GEMMA_LAYERS * 2 * m * n * k
            return nbytes, ops

        def rates(us, ps):
            nbytes, ops = work(ps)
            t_mem, t_tc = nbytes / (hbm * 1e3), ops / (tc * 1e6)  # us at the peaks
            return {"us": round(us, 2), "GBs": round(nbytes / (us * 1e3), 1),
                    "TOPS": round(ops / (us * 1e6), 2), "roofline_frac": round(max(t_mem, t_tc) / us, 4)}

        all_p = range(len(synth.GEMMA_PROJ))
        us_all = timed_graph([call(layer, p) for layer in range(synth.GEMMA_LAYERS) for p in all_p])

        # The same 182 linears with a transformer layer's dependency structure
        # instead of one serial chain: q, k, v on three streams, then o, then
        # gate and up on two streams, then down (fork and join through events
        # inside the one graph). Outputs of parallel branches go to distinct
        # buffers, so the branches share no memory.
        side = [torch.cuda.Stream(device=device) for _ in range(2)]

        def branches(layer, group):
            main = torch.cuda.current_stream()
            for st in side[:len(group) - 1]:
                st.wait_stream(main)
            for st, p in zip([main] + side, group):
                with torch.cuda.stream(st):
                    call(layer, p)()
            for st in side[:len(group) - 1]:
                main.wait_stream(st)

        def layered():
            for layer in range(synth.GEMMA_LAYERS):
                branches(layer, [0, 1, 2])  # q, k, v
                call(layer, 3)()            # o
                branches(layer, [4, 5])     # gate, up
                call(layer, 6)()            # down
        us_dep = timed_graph([layered])

        # All 182 linears as one grouped call (M <= 4 only): persistent
        # launches of up to 64 problems each instead of 182 launches.
        us_grp = None
        if m <= 4:
            probs = [(xs[p], layers[layer][p][0], layers[layer][p][1], None)
                     for layer in range(synth.GEMMA_LAYERS) for p in all_p]
            outs = [torch.empty((m, synth.GEMMA_PROJ[p][2]), dtype=torch.float32, device=device)
                    for p in all_p]
            arr = (native.Problem * len(probs))()
            for i, (x, wp, sw, _) in enumerate(probs):
                n = wp.shape[0]
                y = outs[i % len(outs)]
                arr[i] = native.Problem(x.data_ptr(), wp.data_ptr(), sw.data_ptr(), None, y.data_ptr(),
                                        m, x.shape[1], x.stride(0), wp.stride(0), n, y.stride(0))
            flags = native.flags_for(static_weights=True)

            def grouped():
                rc = native.lib.w4a8_linear_grouped(arr, len(probs), flags,
                                                   native._stream(torch.cuda.current_stream()))
                assert rc == native.OK, rc
            us_grp = timed_graph([grouped])
        per_type = {}
        for p, (nm, _, _) in enumerate(synth.GEMMA_PROJ):
            us_p = timed_graph([call(layer, p) for layer in range(synth.GEMMA_LAYERS)])
            per_type[nm] = rates(us_p, [p])
        print(json.dumps({"workload": "gemma3-1b-shaped stack, 26 layers x 7 linears in one CUDA graph",
                          "M": m, "aggregate": rates(us_all, list(all_p)),
                          "aggregate_layer_dependencies": rates(us_dep, list(all_p)),
                          "aggregate_grouped": rates(us_grp, list(all_p)) if us_grp else None,
                          "per_type": per_type, "call": "w4a8_linear with W4A8_STATIC_WEIGHTS",
                          "note": "aggregate: one serial chain of 182 calls; aggregate_layer_dependencies: "
                                  "q/k/v and gate/up as parallel branches, o and down after them; "
                                  "aggregate_grouped: the 182 independent linears through "
                                  "w4a8_linear_grouped (one launch per 64)"}),
              flush=True)
        del xs, ys, wss


# --------------------------------------------------------------- main ---

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=8.0,
                    help="seconds of CPU work per oracle baseline (decode, prefill sample)")
    ap.add_argument("--workload", choices=["decode", "prefill", "prefill-relu", "sweep", "gemma-stack",
                                           "decode-w8a8", "prefill-w8a8", "decode-zp", "decode-grp", "prefill-grp"],
                    default="decode",
                    help="decode (the default line: decode, with the prefill sub-record), prefill "
                         "(M=2048 K=4096 N=11008) alone, a per-shape sweep of the other workloads, the "
                         "182-linear Gemma3-1B-shaped stack, or the decode / prefill workloads on the "
                         "W8A8, zero-point and group-wise paths")
    ap.add_argument("--no-prefill", action="store_true", help="leave the prefill sub-record out of the default line")
    ap.add_argument("--min-timed-s", type=float, default=MIN_TIMED_S,
                    help="repeat each timed region until this much device time is covered (at least 5 "
                         "repeats); a small value keeps profiler runs short")
    args = ap.parse_args()
    globals()["MIN_TIMED_S"] = max(0.0, args.min_timed_s)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from w4a8_quantized_gemm_channel_b200 import native, synth

    # the CPU baselines run before any GPU work, on rank 0 only, at N = 1
    cpu = cpu_pf = None
    threads = cpu_threads()
    want_prefill = args.workload == "decode" and not args.no_prefill
    if rank == 0 and world == 1:
        if args.workload in ("decode", "prefill", "prefill-relu"):
            if args.workload == "decode":
                gbs, t, steps = oracle_decode_steps(args.cpu_budget, threads)
                cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                       "sample": f"{steps} full decode steps (M = 1, 4, 16; K = N = 4096; every output "
                                 f"channel) on {threads} threads, {t:.2f} s of plain-C oracle work"}
            if want_prefill or args.workload != "decode":
                tops, det = oracle_prefill_rate(args.cpu_budget, threads, synth.prefill_case())
                cpu_pf = {"value": round(tops, 6), "unit": "TOPS", "cores": threads, "kind": "oracle",
                          "sample": f"activation pass over all of X, then the product on {det['channels']} of "
                                    f"{synth.PREFILL_N} output channels (full M and K) in {det['t_sample_s']} s "
                                    f"on {threads} threads; the full-layer rate is extrapolated from that sample"}

    props = torch.cuda.get_device_properties(device)
    if args.workload in ("prefill", "prefill-relu", "prefill-w8a8", "prefill-grp"):
        run_prefill(args, torch, native, synth, device, props, dist, world, rank,
                    relu=args.workload == "prefill-relu", w8=args.workload == "prefill-w8a8", cpu=cpu_pf,
                    grp=args.workload == "prefill-grp")
        return
    if args.workload in ("decode-w8a8", "decode-zp", "decode-grp"):
        run_decode_w8a8(args, torch, native, synth, device, props, dist, world, rank,
                        zp=args.workload == "decode-zp", grp=args.workload == "decode-grp")
        return
    if args.workload == "sweep":
        run_sweep(torch, native, synth, device, props)
        return
    if args.workload == "gemma-stack":
        run_gemma_stack(torch, native, synth, device)
        return

    rec = decode_record(args, torch, native, synth, device, props, dist, world, form="w4")
    line = {"metric": METRIC, "value": rec.pop("value"), "unit": rec.pop("unit"), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": rec.pop("dtype"),
            "data": "synthetic", **rec}
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if want_prefill:
        line["prefill"] = prefill_record(args, torch, native, synth, device, props, dist, world, rank, cpu=cpu_pf)
        line["gpu_launches"] += line["prefill"]["gpu_launches"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
