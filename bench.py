#!/usr/bin/env python
"""Benchmark of the NVFP4 / MXFP8 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass over every row of the hot path, each on its workload
(seeded synthetic inputs, resident in HBM before timing):

  quant1g   a1-a4   amax + NVFP4 quantize (SWIZZLED scales) of bf16 [32768,16384]
  quant1g_sr f4     the same quantize with stochastic rounding of the codes
  gemv      a1,a6-a7  amax(x) + qmv: x [1,4096] bf16, W [14336,4096] pre-quantized
  dequant   a5      NVFP4 dequantize of W [14336,4096] to bf16
  prefill   a1-a4,a8-a9  qqmm op: amax x2, quantize x2 (SWIZZLED), FP4 GEMM 4096^3 -> bf16
  prefill_bwd f1    qqmm backward: amax + quantize of the gradient, column-wise
                    quantizes of W, x and the gradient, dx and dw GEMMs 4096^3
  moe       a10     gather_qmm: 64 experts [1408,2048], 4096 tokens, top-8 -> bf16
  moe_kn    f2      gather_qmm with transpose=False: the moe row's weights stored [E, K, N]
  moe_decode f2     gather_qmm decode (gather_qmv): the same experts, 4 tokens, top-8
  mxfp8     a11-a12 mxfp8 quantize x2 + FP8 GEMM 8192^3 -> bf16
  mxfp4     f3      mxfp4 quantize x2 + FP4 GEMM 8192^3 (mxfp4 mode) -> bf16

The headline ``value`` is the prefill qqmm op in TFLOP/s (2*M*N*K over the
whole op: amaxes, quantizes and GEMM); every row's own metric, time and
roofline are under ``rows``.  L2 (126 MB) is flushed before every row by
writing a 256 MiB buffer and then reading another 256 MiB buffer (the read
evicts the flush's dirty lines, so their write-back to HBM is not charged to
the row's first kernel), outside the row's timed window.  The calls of a row
are captured as one CUDA graph with timing events recorded inside the graph
before the first call and after every call; each timed step replays its own
copy of the graph behind the flush, so neither host-side call overhead nor
the graph's launch latency is inside any window.  A single call timed this
way still carries its own launch and the idle ramp behind the flush, so each
row's roofline kernel is also timed back to back: R launches of that call
over rotating copies of its operands whose footprint exceeds L2 (the
alternative to a flush between timed launches), captured as one graph with
events only around the R launches; the roofline's ``achieved`` is work per
launch over that mean, ``achieved_isolated`` the flushed single call.

Multi-GPU (torchrun, one process per GPU): every rank runs the same step on
its own GPU over its own draw of each workload (seed offset = rank; rank 0
has the workload itself): independent problems, no data-path collective,
weak scaling; the reported time is the max over ranks.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20

# dram__bytes_read.sum + dram__bytes_write.sum per launch of each row's
# dominant kernel, from one ncu capture of that kernel as it is now (the
# summaries under profiles/ give the commands and the other counters).
NCU_TRAFFIC_BYTES = {
    "qqmm_sm100 (nvfp4)": 18959872 + 134656,     # profiles/qqmm_nvfp4_4096x4096x4096.md
    "k_qmv_tc": 33114880 + 0,                    # profiles/qmv_tc_gemv_14336x4096.md
    "gather_qmm": 238368512 + 72332288,          # profiles/gather_qmm_moe_T4096_top8_E64_N1408_K2048.md (k_gather_mma_ts)
    "gather_qmm (kn)": 127801600 + 56908544,     # profiles/gather_qmm_kn_moe_T4096_top8_E64_N1408_K2048.md
    "qqmm_sm100 (mxfp4)": 103694592 + 103843584, # profiles/qqmm_mxfp4_8192x8192x8192.md
    "k_nvfp4_quantize<SR>": 1136302336 + 326791168,  # profiles/quantize_sr_32768x16384.md
    "k_nvfp4_quantize": 1082603008 + 288834048,  # profiles/quantize_nvfp4_32768x16384.md
    "k_gather_qmv": 43878656 + 4864,               # profiles/gather_qmv_decode_T4_top8_E64_N1408_K2048.md
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# rows of the hot path
# ---------------------------------------------------------------------------
class Row:
    """One row of the hot path.  ``calls()`` lists its ABI calls as
    (label, fn) with every output preallocated.  The row is captured as one
    CUDA graph with a timing event recorded inside the graph before the
    first call and after every call (external events: the graph records
    them each replay), so per-call and whole-row device times exclude the
    graph's launch latency.  Each timed step replays its own copy of the
    graph, so no event is overwritten before it is read."""
    name = ""
    launches = 0  # our kernels per run

    def __init__(self, nv, wl, dev, seed_offset):
        self.nv, self.wl, self.dev, self.off = nv, wl, dev, seed_offset
        self.copies = []  # (CUDAGraph, labels, events)
        self.used = []    # copies replayed in the timed region

    def run(self):
        for _, fn in self.calls():
            fn()

    def capture(self, copies):
        self.copies = []
        for _ in range(copies):
            calls = self.calls()
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(calls) + 1)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                evs[0].record()
                for i, (_, fn) in enumerate(calls):
                    fn()
                    evs[i + 1].record()
            self.copies.append((g, [label for label, _ in calls], evs))

    def replay(self, k, timed):
        g = self.copies[k % len(self.copies)][0]
        g.replay()
        if timed:
            self.used.append(k % len(self.copies))

    # The row's roofline call timed back to back: ``b2b()`` returns R
    # callables of that call over rotating copies of its operands whose
    # footprint exceeds L2 (the alternative to an L2 flush between timed
    # launches), captured as one graph with events only around the R launches,
    # so the mean is the kernel's own launch duration with cold operands.
    b2b_label = None
    b2b_kernels = 1  # our kernels per back-to-back call
    b2b_n = 0

    def b2b(self):
        return None

    def capture_b2b(self, copies):
        self.b2b_copies, self.b2b_used = [], []
        fns = self.b2b()
        # the graphs hold raw pointers into the operand copies the callables
        # close over: keep them alive for as long as the graphs are replayed
        self.b2b_fns = fns
        if not fns:
            return
        self.b2b_n = len(fns)
        for _ in range(copies):
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                evs[0].record()
                for fn in fns:
                    fn()
                evs[1].record()
            self.b2b_copies.append((g, evs))

    def replay_b2b(self, k, timed):
        if not self.b2b_copies:
            return
        self.b2b_copies[k % len(self.b2b_copies)][0].replay()
        if timed:
            self.b2b_used.append(k % len(self.b2b_copies))

    def b2b_ms(self):
        """Mean ms per launch of the back-to-back call, or None."""
        if not self.b2b_used:
            return None
        tot = sum(self.b2b_copies[k][1][0].elapsed_time(self.b2b_copies[k][1][1]) for k in self.b2b_used)
        return tot / len(self.b2b_used) / self.b2b_n

    def times(self):
        """Mean ms per call and per row over the timed replays."""
        per, row = {}, 0.0
        for k in self.used:
            _, labels, evs = self.copies[k]
            for i, label in enumerate(labels):
                per[label] = per.get(label, 0.0) + evs[i].elapsed_time(evs[i + 1])
            row += evs[0].elapsed_time(evs[-1])
        n = max(1, len(self.used))
        return {k: v / n for k, v in per.items()}, row / n


def _rot(fns, n):
    """n calls cycling through the callables fns (one per operand copy)."""
    return [fns[i % len(fns)] for i in range(n)]


class Quant1G(Row):
    name, launches = "quant1g", 2
    b2b_label = "quantize"

    def b2b(self):  # 1 GiB of input per call: larger than L2 on its own
        return [lambda: self.nv.nvfp4_quantize(self.x, self.g, "swizzled", self.codes, self.scales)] * 2

    def setup(self):
        self.x = self.wl.make("quant1g", device=self.dev, seed_offset=self.off)["x"]
        R, K = self.x.shape
        self.g = torch.empty(1, dtype=torch.float32, device=self.dev)
        self.codes = torch.empty(R, K // 8, dtype=torch.int32, device=self.dev)
        self.scales = torch.empty(self.nv.scale_shape(R, K // 16, "swizzled"), dtype=torch.uint8, device=self.dev)
        self.units = R * K
        # algorithmic bytes of the quantize kernel: read x, write codes + scales
        self.bytes_q = R * K * 2 + R * K // 2 + self.scales.numel()

    def calls(self):
        return [("amax", lambda: self.nv.amax(self.x, self.g)),
                ("quantize", lambda: self.nv.nvfp4_quantize(self.x, self.g, "swizzled", self.codes, self.scales))]

    def report(self, ms, row_ms, peaks):
        q = ms["quantize"]
        return {"metric": "nvfp4 quantize GB/s", "unit": "GB/s", "value": self.bytes_q / q / 1e6,
                "ms": ms, "roofline": {"bound": "hbm", "kernel": "k_nvfp4_quantize", "achieved": self.bytes_q / q / 1e6,
                                       "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                       "frac": self.bytes_q / q / 1e6 / peaks["hbm_gbs"],
                                       "frac_of_8tbs": self.bytes_q / q / 1e6 / 8000.0,
                                       "algorithmic_bytes": self.bytes_q}}


class Quant1GSR(Quant1G):
    """The 1 GiB quantize with stochastic rounding of the codes (Philox4x32-10
    bits per element, seed fixed): the same bytes as quant1g."""
    name, launches = "quant1g_sr", 2

    def b2b(self):
        return [lambda: self.nv.nvfp4_quantize_sr(self.x, self.g, 20261202, "swizzled", self.codes, self.scales)] * 2

    def calls(self):
        return [("amax", lambda: self.nv.amax(self.x, self.g)),
                ("quantize", lambda: self.nv.nvfp4_quantize_sr(self.x, self.g, 20261202, "swizzled", self.codes,
                                                               self.scales))]

    def report(self, ms, row_ms, peaks):
        r = super().report(ms, row_ms, peaks)
        r["metric"] = "nvfp4 quantize (stochastic rounding) GB/s"
        r["roofline"]["kernel"] = "k_nvfp4_quantize<SR>"
        return r


class Gemv(Row):
    name, launches = "gemv", 2
    b2b_label = "qmv"

    def b2b(self):  # six copies of the 33 MB weight (198 MB), two passes
        cps = [(self.wc.clone(), self.ws.clone()) for _ in range(6)]
        return _rot([lambda c=c: self.nv.qmv(self.x, c[0], c[1], self.g_x, self.g_w, self.y) for c in cps], 12)

    def setup(self):
        d = self.wl.make("gemv", device=self.dev, seed_offset=self.off)
        self.x, w = d["x"], d["w"]
        self.g_x = torch.empty(1, dtype=torch.float32, device=self.dev)
        self.g_w = self.nv.amax(w)
        self.wc, self.ws = self.nv.nvfp4_quantize(w, self.g_w, "linear")
        del w
        self.N, self.K = self.wc.shape[0], self.x.shape[1]
        self.y = torch.empty(1, self.N, dtype=torch.bfloat16, device=self.dev)
        self.bytes = self.wc.numel() * 4 + self.ws.numel() + self.x.numel() * 2 + self.y.numel() * 2

    def calls(self):
        return [("amax", lambda: self.nv.amax(self.x, self.g_x)),
                ("qmv", lambda: self.nv.qmv(self.x, self.wc, self.ws, self.g_x, self.g_w, self.y))]

    def report(self, ms, row_ms, peaks):
        q = ms["qmv"]
        gbs = self.bytes / q / 1e6
        return {"metric": "qmv GB/s", "unit": "GB/s", "value": gbs, "ms": ms,
                "roofline": {"bound": "hbm", "kernel": "k_qmv_tc", "achieved": gbs, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "frac_of_8tbs": gbs / 8000.0,
                             "algorithmic_bytes": self.bytes}}


class GemvChain(Gemv):
    """The decode GEMV as a chain of calls with fixed weights (qmv_pdl: each
    call streams its weight while the previous call drains); same workload
    and bytes as the gemv row.  Its weight copies are written in set-up and
    synchronized before any qmv_pdl call, as the entry point requires."""
    name = "gemv_chain"

    def b2b(self):
        cps = [(self.wc.clone(), self.ws.clone()) for _ in range(6)]
        torch.cuda.synchronize()
        return _rot([lambda c=c: self.nv.qmv(self.x, c[0], c[1], self.g_x, self.g_w, self.y, pdl=True)
                     for c in cps], 12)

    def setup(self):
        super().setup()
        torch.cuda.synchronize()

    def calls(self):
        return [("amax", lambda: self.nv.amax(self.x, self.g_x)),
                ("qmv", lambda: self.nv.qmv(self.x, self.wc, self.ws, self.g_x, self.g_w, self.y, pdl=True))]

    def report(self, ms, row_ms, peaks):
        r = super().report(ms, row_ms, peaks)
        r["metric"] = "qmv GB/s (qmv_pdl chain)"
        r["roofline"]["kernel"] = "k_qmv_tc<PDL>"
        return r


class Dequant(Row):
    name, launches = "dequant", 1
    b2b_label = "dequantize"

    def b2b(self):  # three copies of the 33 MB input, 117 MB written per call
        cps = [(self.wc.clone(), self.ws.clone()) for _ in range(3)]
        return _rot([lambda c=c: self.nv.nvfp4_dequantize(c[0], c[1], self.g, "linear", out=self.out)
                     for c in cps], 6)

    def setup(self):
        w = self.wl.make("gemv", device=self.dev, seed_offset=self.off)["w"]
        g = self.nv.amax(w)
        self.g = g
        self.wc, self.ws = self.nv.nvfp4_quantize(w, g, "linear")
        self.out = torch.empty_like(w)
        self.bytes = self.wc.numel() * 4 + self.ws.numel() + w.numel() * 2
        del w

    def calls(self):
        return [("dequantize", lambda: self.nv.nvfp4_dequantize(self.wc, self.ws, self.g, "linear",
                                                                torch.bfloat16, out=self.out))]

    def report(self, ms, row_ms, peaks):
        q = ms["dequantize"]
        gbs = self.bytes / q / 1e6
        return {"metric": "nvfp4 dequantize GB/s", "unit": "GB/s", "value": gbs, "ms": ms,
                "roofline": {"bound": "hbm", "kernel": "k_nvfp4_dequantize", "achieved": gbs,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                             "algorithmic_bytes": self.bytes}}


class Prefill(Row):
    name, launches = "prefill", 3
    b2b_label = "gemm"

    def b2b(self):  # eight copies of the quantized operands (8 x 18.9 MB), two passes
        cps = [(self.xc.clone(), self.xs.clone(), self.wc.clone(), self.ws.clone()) for _ in range(8)]
        return _rot([lambda c=c: self.nv.qqmm(c[0], c[1], c[2], c[3], self.K, "nvfp4", self.g_x, self.g_w,
                                              out=self.y) for c in cps], 16)

    def setup(self):
        d = self.wl.make("prefill", device=self.dev, seed_offset=self.off)
        self.x, self.w = d["x"], d["w"]
        self.M, self.K = self.x.shape
        self.N = self.w.shape[0]
        self.g = torch.empty(2, dtype=torch.float32, device=self.dev)  # g_x, g_w
        self.g_x, self.g_w = self.g[0:1], self.g[1:2]
        mk = lambda r: (torch.empty(r, self.K // 8, dtype=torch.int32, device=self.dev),
                        torch.empty(self.nv.scale_shape(r, self.K // 16, "swizzled"), dtype=torch.uint8,
                                    device=self.dev))
        self.xc, self.xs = mk(self.M)
        self.wc, self.ws = mk(self.N)
        self.y = torch.empty(self.M, self.N, dtype=torch.bfloat16, device=self.dev)
        self.flop = 2 * self.M * self.N * self.K
        # probe: raises if the GEMM kernel is not available
        self.nv.nvfp4_quantize(self.x[:128], None, "swizzled")
        self.nv.qqmm(self.xc[:128], self.xs[:128], self.wc[:128], self.ws[:128], self.K, "nvfp4",
                     out=self.y[:128, :128].contiguous())

    def calls(self):
        nv = self.nv
        # the steps of nvfp4.qqmm_raw: both amaxes in one launch, both
        # quantizations in one launch, the GEMM
        return [("amax", lambda: nv.amax_multi([self.x, self.w], self.g)),
                ("quantize", lambda: nv.nvfp4_quantize_multi([(self.x, self.g_x, "swizzled", self.xc, self.xs),
                                                              (self.w, self.g_w, "swizzled", self.wc, self.ws)])),
                ("gemm", lambda: nv.qqmm(self.xc, self.xs, self.wc, self.ws, self.K, "nvfp4", self.g_x, self.g_w,
                                         out=self.y))]

    def report(self, ms, row_ms, peaks):
        total = row_ms  # the whole op: quantize x and W, GEMM, as one graph
        fp4_peak = peaks["bf16_tflops"] * 4.0  # nominal dense fp4 : bf16 = 9 : 2.25
        tf = self.flop / ms["gemm"] / 1e9
        return {"metric": "qqmm FP4 TFLOP/s", "unit": "TFLOP/s", "value": self.flop / total / 1e9, "ms": ms,
                "roofline": {"bound": "tensor", "kernel": "qqmm_sm100 (nvfp4)", "achieved": tf, "peak": fp4_peak,
                             "unit": "TFLOP/s", "frac": tf / fp4_peak, "algorithmic_flop": self.flop,
                             "peak_note": "measured bf16 burst x 4 (nominal fp4:bf16 ratio)"}}


class PrefillBwd(Row):
    """Backward pass of the prefill qqmm (QQMatmul::vjp, NVFP4 with global
    scales): amax of the upstream gradient, its row-wise and column-wise
    quantization, column-wise quantization of W and x, and the dx and dw
    GEMMs (4096^3 each)."""
    name, launches = "prefill_bwd", 7
    b2b_label = "gemm_dx"

    def b2b(self):  # eight copies of dx's quantized operands, two passes
        cps = [tuple(t.clone() for t in (*self.cq, *self.wtq)) for _ in range(8)]
        return _rot([lambda c=c: self.nv.qqmm(*c, self.N, "nvfp4", self.g_c, self.g_w, out=self.dx)
                     for c in cps], 16)

    def setup(self):
        d = self.wl.make("prefill_bwd", device=self.dev, seed_offset=self.off)
        self.x, self.w, self.c = d["x"], d["w"], d["cotan"]
        M, K = self.x.shape
        N = self.w.shape[0]
        self.M, self.N, self.K = M, N, K
        nv, dev = self.nv, self.dev
        self.g_x, self.g_w = nv.amax(self.x), nv.amax(self.w)
        self.g_c = torch.empty(1, dtype=torch.float32, device=dev)
        q = lambda r, k: (torch.empty(r, k // 8, dtype=torch.int32, device=dev),
                          torch.empty(nv.scale_shape(r, k // 16, "swizzled"), dtype=torch.uint8, device=dev))
        self.cq, self.wtq, self.ctq, self.xtq = q(M, N), q(K, N), q(N, M), q(K, M)
        self.dx = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        self.dw = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        self.flop = 2 * (2 * M * N * K)

    def calls(self):
        nv = self.nv
        return [("amax_cotan", lambda: nv.amax(self.c, self.g_c)),
                ("quantize_cotan", lambda: nv.nvfp4_quantize(self.c, self.g_c, "swizzled", *self.cq)),
                ("quantize_wT", lambda: nv.nvfp4_quantize_columnwise(self.w, self.g_w, "swizzled", *self.wtq)),
                ("gemm_dx", lambda: nv.qqmm(*self.cq, *self.wtq, self.N, "nvfp4", self.g_c, self.g_w, out=self.dx)),
                ("quantize_cotanT", lambda: nv.nvfp4_quantize_columnwise(self.c, self.g_c, "swizzled", *self.ctq)),
                ("quantize_xT", lambda: nv.nvfp4_quantize_columnwise(self.x, self.g_x, "swizzled", *self.xtq)),
                ("gemm_dw", lambda: nv.qqmm(*self.ctq, *self.xtq, self.M, "nvfp4", self.g_c, self.g_x, out=self.dw))]

    def report(self, ms, row_ms, peaks):
        fp4_peak = peaks["bf16_tflops"] * 4.0
        col_bytes = 2 * self.M * self.K + self.M * self.K // 2 + self.M * self.K // 16  # one 4096^2 bf16 operand
        return {"metric": "qqmm backward FP4 TFLOP/s", "unit": "TFLOP/s", "value": self.flop / row_ms / 1e9, "ms": ms,
                "columnwise_quantize_gbs": col_bytes / ms["quantize_xT"] / 1e6,
                "roofline": {"bound": "tensor", "kernel": "qqmm_sm100 (nvfp4)",
                             "achieved": (self.flop / 2) / ms["gemm_dx"] / 1e9, "peak": fp4_peak, "unit": "TFLOP/s",
                             "frac": (self.flop / 2) / ms["gemm_dx"] / 1e9 / fp4_peak,
                             "algorithmic_flop": self.flop // 2,
                             "peak_note": "measured bf16 burst x 4 (nominal fp4:bf16 ratio)"}}


class Moe(Row):
    """The MoE config through gather_qmm with a staged workspace: routing,
    the staged copy of the routed x rows, the SM-pair tensor-core kernel."""
    name, launches = "moe", 3  # k_route + k_stage_x + k_gather_mma_ts
    b2b_label = "gather_qmm"
    b2b_kernels = 3
    b2b_transpose = True

    def b2b(self):  # two copies of the 108 MB expert weights, alternating
        cps = [(self.wc, self.ws), (self.wc.clone(), self.ws.clone())]
        return _rot([lambda c=c: self.nv.gather_qmm(self.x, c[0], c[1], self.g, self.idx, self.ws_buf, self.y,
                                                    transpose=self.b2b_transpose) for c in cps], 4)

    def setup(self):
        d = self.wl.make("moe", device=self.dev, seed_offset=self.off)
        self.x, w, self.idx = d["x"], d["w"], d["idx"]
        E, N, K = w.shape
        self.E, self.N, self.K = E, N, K
        self.g = torch.stack([self.nv.amax(w[e]) for e in range(E)]).view(E)
        wc, ws = [], []
        for e in range(E):
            c, s = self.nv.nvfp4_quantize(w[e], self.g[e:e + 1], "linear")
            wc.append(c)
            ws.append(s)
        self.wc, self.ws = torch.stack(wc), torch.stack(ws)
        del w, wc, ws
        T, topk = self.idx.shape
        self.T, self.topk = T, topk
        self.ws_buf = torch.empty(self.nv.gather_qmm_staged_workspace_size(T, topk, E, K), dtype=torch.uint8,
                                  device=self.dev)
        self.y = torch.empty(T, topk, N, dtype=torch.bfloat16, device=self.dev)
        self.flop = 2 * T * topk * N * K
        self.bytes = self.wc.numel() * 4 + self.ws.numel() + self.x.numel() * 2 + self.y.numel() * 2 + self.idx.numel() * 4
        self.nv.gather_qmm(self.x[:16], self.wc, self.ws, self.g, self.idx[:16].contiguous())

    def calls(self):
        return [("gather_qmm", lambda: self.nv.gather_qmm(self.x, self.wc, self.ws, self.g, self.idx,
                                                          self.ws_buf, self.y))]

    def report(self, ms, row_ms, peaks):
        t = ms["gather_qmm"]
        tf = self.flop / t / 1e9
        return {"metric": "gather_qmm TFLOP/s", "unit": "TFLOP/s", "value": tf, "ms": ms,
                "gbs": self.bytes / t / 1e6,
                "roofline": {"bound": "tensor", "kernel": "gather_qmm", "achieved": tf, "peak": peaks["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"], "algorithmic_flop": self.flop,
                             "hbm_frac": self.bytes / t / 1e6 / peaks["hbm_gbs"], "algorithmic_bytes": self.bytes}}


class MoeKN(Moe):
    """The MoE config with the expert weights stored [E, K, N] and quantized
    along N (gather_qmm with transpose=False): same tokens, routing and
    per-expert global scales as the moe row."""
    name, launches = "moe_kn", 2  # k_route + k_gather_mma<true>
    b2b_kernels = 2
    b2b_transpose = False

    def setup(self):
        d = self.wl.make("moe", device=self.dev, seed_offset=self.off)
        self.x, w, self.idx = d["x"], d["w"], d["idx"]
        E, N, K = w.shape
        self.E, self.N, self.K = E, N, K
        wt = w.transpose(1, 2).contiguous()  # [E, K, N]
        del w
        self.g = torch.stack([self.nv.amax(wt[e]) for e in range(E)]).view(E)
        wc, ws = [], []
        for e in range(E):
            c, s = self.nv.nvfp4_quantize(wt[e], self.g[e:e + 1], "linear")
            wc.append(c)
            ws.append(s)
        self.wc, self.ws = torch.stack(wc), torch.stack(ws)
        del wt, wc, ws
        T, topk = self.idx.shape
        self.T, self.topk = T, topk
        self.ws_buf = torch.empty(self.nv.gather_qmm_workspace_size(T, topk, E), dtype=torch.uint8, device=self.dev)
        self.y = torch.empty(T, topk, N, dtype=torch.bfloat16, device=self.dev)
        self.flop = 2 * T * topk * N * K
        self.bytes = self.wc.numel() * 4 + self.ws.numel() + self.x.numel() * 2 + self.y.numel() * 2 + self.idx.numel() * 4
        self.nv.gather_qmm(self.x[:16], self.wc, self.ws, self.g, self.idx[:16].contiguous(), transpose=False)

    def calls(self):
        return [("gather_qmm", lambda: self.nv.gather_qmm(self.x, self.wc, self.ws, self.g, self.idx,
                                                          self.ws_buf, self.y, transpose=False))]

    def report(self, ms, row_ms, peaks):
        r = super().report(ms, row_ms, peaks)
        r["metric"] = "gather_qmm (transpose=False) TFLOP/s"
        r["roofline"]["kernel"] = "gather_qmm (kn)"
        return r


class MoeDecode(Row):
    """Decode-time MoE (the gather_qmv path): the MoE config's 64 experts
    [1408, 2048], 4 tokens routed top-8 (tokens 0-3 of the MoE routing)."""
    name, launches = "moe_decode", 2
    b2b_label = "gather_qmm"
    b2b_kernels = 2  # routing + the decode kernel

    def b2b(self):  # four copies of the experts' weights (the call reads the routed ones)
        cps = [(self.wc.clone(), self.ws.clone()) for _ in range(4)]
        return _rot([lambda c=c: self.nv.gather_qmm(self.x, c[0], c[1], self.g, self.idx, self.ws_buf, self.y)
                     for c in cps], 8)

    def setup(self):
        d = self.wl.make("moe", device=self.dev, seed_offset=self.off)
        x, w, idx = d["x"], d["w"], d["idx"]
        E, N, K = w.shape
        self.E, self.N, self.K = E, N, K
        self.g = torch.stack([self.nv.amax(w[e]) for e in range(E)]).view(E)
        wc, ws = [], []
        for e in range(E):
            c, s = self.nv.nvfp4_quantize(w[e], self.g[e:e + 1], "linear")
            wc.append(c)
            ws.append(s)
        self.wc, self.ws = torch.stack(wc), torch.stack(ws)
        del w, wc, ws
        self.T = 4
        self.x = x[:self.T].contiguous()
        self.idx = idx[:self.T].contiguous()
        self.topk = self.idx.shape[1]
        self.ws_buf = torch.empty(self.nv.gather_qmm_workspace_size(self.T, self.topk, E), dtype=torch.uint8,
                                  device=self.dev)
        self.y = torch.empty(self.T, self.topk, N, dtype=torch.bfloat16, device=self.dev)
        used = int(torch.unique(self.idx).numel())  # each routed expert's weight is read once
        self.experts_read = used
        self.bytes = used * (N * K // 2 + N * K // 16) + self.x.numel() * 2 + self.y.numel() * 2 + self.idx.numel() * 4

    def calls(self):
        return [("gather_qmm", lambda: self.nv.gather_qmm(self.x, self.wc, self.ws, self.g, self.idx,
                                                          self.ws_buf, self.y))]

    def report(self, ms, row_ms, peaks):
        t = ms["gather_qmm"]
        gbs = self.bytes / t / 1e6
        return {"metric": "gather_qmm decode GB/s", "unit": "GB/s", "value": gbs, "ms": ms,
                "experts_read": self.experts_read,
                "roofline": {"bound": "hbm", "kernel": "k_gather_qmv", "achieved": gbs, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes": self.bytes}}


class Mxfp8(Row):
    name, launches = "mxfp8", 3
    b2b_label = "gemm"

    def b2b(self):  # 132 MB of operands per call: larger than L2 on its own
        return [lambda: self.nv.qqmm(self.xc, self.xs, self.wc, self.ws, self.K, "mxfp8", out=self.y)] * 2

    def setup(self):
        d = self.wl.make("mxfp8", device=self.dev, seed_offset=self.off)
        self.x, self.w = d["x"], d["w"]
        self.M, self.K = self.x.shape
        self.N = self.w.shape[0]
        mk = lambda r: (torch.empty(r, self.K // 4, dtype=torch.int32, device=self.dev),
                        torch.empty(self.nv.scale_shape(r, self.K // 32, "swizzled"), dtype=torch.uint8,
                                    device=self.dev))
        self.xc, self.xs = mk(self.M)
        self.wc, self.ws = mk(self.N)
        self.y = torch.empty(self.M, self.N, dtype=torch.bfloat16, device=self.dev)
        self.flop = 2 * self.M * self.N * self.K
        self.nv.qqmm(self.xc[:128], self.xs[:128], self.wc[:128], self.ws[:128], self.K, "mxfp8",
                     out=self.y[:128, :128].contiguous())

    def calls(self):
        nv = self.nv
        return [("quantize_x", lambda: nv.mxfp8_quantize(self.x, "swizzled", self.xc, self.xs)),
                ("quantize_w", lambda: nv.mxfp8_quantize(self.w, "swizzled", self.wc, self.ws)),
                ("gemm", lambda: nv.qqmm(self.xc, self.xs, self.wc, self.ws, self.K, "mxfp8", out=self.y))]

    def report(self, ms, row_ms, peaks):
        fp8_peak = peaks["bf16_tflops"] * 2.0
        tf = self.flop / ms["gemm"] / 1e9
        return {"metric": "mxfp8 qqmm TFLOP/s", "unit": "TFLOP/s", "value": self.flop / row_ms / 1e9,
                "ms": ms, "roofline": {"bound": "tensor", "kernel": "qqmm_sm100 (mxfp8)", "achieved": tf,
                                       "peak": fp8_peak, "unit": "TFLOP/s", "frac": tf / fp8_peak,
                                       "peak_note": "measured bf16 burst x 2 (nominal fp8:bf16 ratio)"}}


class Mxfp4(Row):
    """The MXFP4 mode on the MXFP8 row's operands (x, W [8192, 8192] bf16
    N(0,1)): two MXFP4 quantizes (e8m0 scales per 32, SWIZZLED) and the
    block-scaled GEMM on the FP4 tensor pipe."""
    name, launches = "mxfp4", 3
    b2b_label = "gemm"

    def b2b(self):  # two copies of the 68 MB operands, alternating
        cps = [(self.xc, self.xs, self.wc, self.ws), tuple(t.clone() for t in (self.xc, self.xs, self.wc, self.ws))]
        return _rot([lambda c=c: self.nv.qqmm(*c, self.K, "mxfp4", out=self.y) for c in cps], 4)

    def setup(self):
        d = self.wl.make("mxfp4", device=self.dev, seed_offset=self.off)
        self.x, self.w = d["x"], d["w"]
        self.M, self.K = self.x.shape
        self.N = self.w.shape[0]
        mk = lambda r: (torch.empty(r, self.K // 8, dtype=torch.int32, device=self.dev),
                        torch.empty(self.nv.scale_shape(r, self.K // 32, "swizzled"), dtype=torch.uint8,
                                    device=self.dev))
        self.xc, self.xs = mk(self.M)
        self.wc, self.ws = mk(self.N)
        self.y = torch.empty(self.M, self.N, dtype=torch.bfloat16, device=self.dev)
        self.flop = 2 * self.M * self.N * self.K
        self.bytes_q = self.M * self.K * 2 + self.M * self.K // 2 + self.M * self.K // 32
        self.nv.qqmm(self.xc[:128], self.xs[:128], self.wc[:128], self.ws[:128], self.K, "mxfp4",
                     out=self.y[:128, :128].contiguous())

    def calls(self):
        nv = self.nv
        return [("quantize_x", lambda: nv.mxfp4_quantize(self.x, "swizzled", self.xc, self.xs)),
                ("quantize_w", lambda: nv.mxfp4_quantize(self.w, "swizzled", self.wc, self.ws)),
                ("gemm", lambda: nv.qqmm(self.xc, self.xs, self.wc, self.ws, self.K, "mxfp4", out=self.y))]

    def report(self, ms, row_ms, peaks):
        fp4_peak = peaks["bf16_tflops"] * 4.0
        tf = self.flop / ms["gemm"] / 1e9
        return {"metric": "mxfp4 qqmm TFLOP/s", "unit": "TFLOP/s", "value": self.flop / row_ms / 1e9,
                "ms": ms, "quantize_gbs": self.bytes_q / ms["quantize_x"] / 1e6,
                "roofline": {"bound": "tensor", "kernel": "qqmm_sm100 (mxfp4)", "achieved": tf,
                             "peak": fp4_peak, "unit": "TFLOP/s", "frac": tf / fp4_peak,
                             "peak_note": "measured bf16 burst x 4 (nominal fp4:bf16 ratio)"}}


ROWS = [Quant1G, Quant1GSR, Gemv, GemvChain, Dequant, Prefill, PrefillBwd, Moe, MoeKN, MoeDecode, Mxfp8, Mxfp4]


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n_gpus != world:
        raise SystemExit(f"--gpus {n_gpus} but {world} process(es): launch N > 1 with torchrun "
                         f"--nproc-per-node N (one process per GPU)")
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, v):
    """Largest value of `v` over all ranks (device timings: the slowest rank
    sets the job's time).  Works on NCCL (CUDA tensor) and gloo (CPU)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job(world, work_per_rank, ms_slowest):
    """Weak scaling: every rank solves its own problem of `work_per_rank`
    units; the job's throughput is all ranks' work over the slowest time."""
    return world * work_per_rank / ms_slowest


def e2e_prefill(nv, row, steps):
    """The headline metric end to end through the public API with HOST
    buffers: pinned bf16 x and W copied in, the qqmm op, y copied out."""
    xh = row.x.cpu().pin_memory()
    wh = row.w.cpu().pin_memory()
    yh = torch.empty(row.M, row.N, dtype=torch.bfloat16).pin_memory()
    xd, wd = torch.empty_like(row.x), torch.empty_like(row.w)

    def once():
        xd.copy_(xh, non_blocking=True)
        wd.copy_(wh, non_blocking=True)
        nv.qqmm_raw(xd, wd, out=row.y, buffers=(row.g, row.xc, row.xs, row.wc, row.ws))
        yh.copy_(row.y, non_blocking=True)

    for _ in range(2):
        once()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        once()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    return {"ms": ms, "work": row.flop / 1e9, "unit": "TFLOP/s",
            "h2d_bytes_per_step": xh.numel() * 2 + wh.numel() * 2, "d2h_bytes_per_step": yh.numel() * 2}


def e2e_gemv(nv, row, steps):
    xh = row.x.cpu().pin_memory()
    yh = torch.empty(1, row.N, dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(row.x)

    def once():
        xd.copy_(xh, non_blocking=True)
        g = nv.amax(xd, row.g_x)
        nv.qmv(xd, row.wc, row.ws, g, row.g_w, row.y)
        yh.copy_(row.y, non_blocking=True)

    for _ in range(3):
        once()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        once()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    return {"ms": ms, "work": row.bytes / 1e6, "unit": "GB/s", "h2d_bytes_per_step": xh.numel() * 2,
            "d2h_bytes_per_step": yh.numel() * 2}


def cpu_baseline_prefill(sample_rows=16, d=None):
    """The oracle as it stands on a bounded sample of the prefill qqmm op:
    amax of x and W, quantize of `sample_rows` rows of x and all of W, exact
    decode, float64 matmul.  Reported in TFLOP/s of the sampled outputs;
    `d` is the workload's inputs when the caller already drew them."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    from oracle import oracle as orc
    orc.build()
    if d is None:
        d = workloads.make("prefill", device="cpu")
    x = d["x"][:sample_rows].contiguous().view(torch.int16).numpy().view(np.uint16)
    wfull = d["w"].contiguous().view(torch.int16).numpy().view(np.uint16)
    xfull = d["x"].contiguous().view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    gx, gw = orc.amax(xfull, "bf16"), orc.amax(wfull, "bf16")
    xq, xs = orc.nvfp4_quantize(x, "bf16", gx)
    wq, ws = orc.nvfp4_quantize(wfull, "bf16", gw)
    orc.qqmm(xq, xs, wq, ws, "nvfp4", gx, gw, "bf16")
    dt = time.perf_counter() - t0
    flop = 2 * sample_rows * wfull.shape[0] * wfull.shape[1]
    threads = 1
    try:
        from threadpoolctl import threadpool_info
        threads = max([1] + [i.get("num_threads", 1) for i in threadpool_info()])
    except Exception:
        pass
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "seconds": dt,
            "sample": f"prefill qqmm op on {sample_rows} of 4096 rows of x (full W quantized, full amaxes); "
                      f"element steps single-threaded C, contraction numpy float64 ({threads} BLAS threads)"}


def cpu_baseline_rows(quant_rows=256, gemv_rows=2048):
    """The oracle as it stands on two more rows of the hot path, on this
    host's cores, each on a bounded slice of its config: the NVFP4 quantize
    on ``quant_rows`` of the 1 GiB config's 32768 rows, and the qmv decode
    GEMV (quantize-dequantize of x, exact weight decode, float64 sum) on
    ``gemv_rows`` of the weight's 14336 rows; GB/s of the slice.  Element
    steps are single-threaded C."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    from oracle import oracle as orc
    orc.build()
    out = {}
    xq = workloads.normal((quant_rows, 16384), 1.0, 10, torch.bfloat16, "cpu")
    xr = xq.contiguous().view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    g = orc.amax(xr, "bf16")
    orc.nvfp4_quantize(xr, "bf16", g)
    dt = time.perf_counter() - t0
    nbytes = quant_rows * 16384 * (2 + 0.5 + 1 / 16)
    out["quant1g"] = {"value": nbytes / dt / 1e9, "unit": "GB/s", "seconds": dt,
                      "sample": f"amax + NVFP4 quantize of {quant_rows} of 32768 rows of the 1 GiB config"}
    d = workloads.make("gemv", device="cpu")
    x = d["x"].contiguous().view(torch.int16).numpy().view(np.uint16)
    w = d["w"][:gemv_rows].contiguous().view(torch.int16).numpy().view(np.uint16)
    gw = orc.amax(w, "bf16")
    wc, ws = orc.nvfp4_quantize(w, "bf16", gw)
    t0 = time.perf_counter()
    gx = orc.amax(x, "bf16")
    orc.qmv(x, "bf16", gx, wc, ws, gw)
    dt = time.perf_counter() - t0
    nbytes = wc.nbytes + ws.nbytes + x.nbytes + 2 * w.shape[0]
    out["gemv"] = {"value": nbytes / dt / 1e9, "unit": "GB/s", "seconds": dt,
                   "sample": f"qmv of the decode config on {gemv_rows} of 14336 weight rows "
                             "(weight pre-quantized, as on the GPU)"}
    return out


def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4 as nv, workloads as wl
    if rank == 0:
        build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.fill_(1.0)                       # write a buffer larger than L2
        torch.sum(flush_rd, dim=0, out=flush_sum)  # read one: L2 holds clean lines only
    rows, unavailable = [], {}
    for cls in ROWS:
        if args.rows and cls.name not in args.rows:
            continue
        r = cls(nv, wl, dev, rank)
        try:
            r.setup()
            torch.cuda.synchronize()
            rows.append(r)
        except nv.Nvfp4Error as e:
            unavailable[cls.name] = str(e)
            torch.cuda.synchronize()
    if not rows:
        raise SystemExit("no row of the hot path is available")

    for _ in range(2):  # eager calls first: one-time set-up of every ABI call
        for r in rows:
            r.run()
    torch.cuda.synchronize()
    for r in rows:
        r.capture(args.steps)
        r.capture_b2b(args.steps)
    torch.cuda.synchronize()

    def step(k, timed):
        for r in rows:
            flush_l2()  # outside the rows' timed windows
            r.replay(k, timed)
            r.replay_b2b(k, timed)

    for k in range(args.warmup):
        step(k, False)
    torch.cuda.synchronize()
    barrier(world)
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    s_all, e_all = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    s_all.record()
    for k in range(args.steps):
        step(k, True)
    e_all.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clocks = clk.stop()
    barrier(world)
    ms_step = max_over_ranks(world, s_all.elapsed_time(e_all) / args.steps)
    reports = {}
    for r in rows:
        per, row_ms = r.times()
        per = {k: max_over_ranks(world, v) for k, v in per.items()}
        row_ms = max_over_ranks(world, row_ms)
        reports[r.name] = r.report(per, row_ms, peaks)
        reports[r.name]["row_ms"] = row_ms
        rf = reports[r.name].get("roofline")
        t_b2b = r.b2b_ms()
        if t_b2b is not None:
            t_b2b = max_over_ranks(world, t_b2b)
            reports[r.name]["b2b_ms"] = t_b2b
        if rf is not None and t_b2b is not None and r.b2b_label in per:
            # the kernel's own launch duration: back to back, cold operands
            ratio = per[r.b2b_label] / t_b2b
            rf["achieved_isolated"] = rf["achieved"]
            rf["achieved"] = rf["achieved"] * ratio
            rf["frac"] = rf["achieved"] / rf["peak"]
            if "hbm_frac" in rf:
                rf["hbm_frac"] = rf["hbm_frac"] * ratio
            rf["kernel_ms"] = t_b2b
            rf["timing"] = (f"'{r.b2b_label}' launched {r.b2b_n} times back to back over operand copies whose "
                            f"footprint exceeds L2; CUDA events around the launches; achieved_isolated: the same "
                            f"call timed alone after an L2 flush")
        if rf is not None:
            rf["traffic"] = NCU_TRAFFIC_BYTES.get(rf.get("kernel"))
    head_row = "prefill" if "prefill" in reports else ("gemv" if "gemv" in reports else rows[0].name)
    head = reports[head_row]
    e2e = None
    byname = {r.name: r for r in rows}
    if head_row == "prefill":
        e2e = e2e_prefill(nv, byname["prefill"], max(3, args.steps))
    elif head_row == "gemv":
        e2e = e2e_gemv(nv, byname["gemv"], max(10, args.steps))
    if e2e is not None:
        # every rank solves its own problem: whole-job work / slowest rank
        ms_e2e = max_over_ranks(world, e2e.pop("ms"))
        e2e = {"value": whole_job(world, e2e.pop("work"), ms_e2e), **e2e, "ms_per_step": ms_e2e}
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline_prefill()
            cpu["rows"] = cpu_baseline_rows()
            if head_row != "prefill":
                cpu["note"] = "headline row is not prefill; baseline of the prefill op shown"
        roof = dict(head["roofline"])
        roof["traffic"] = NCU_TRAFFIC_BYTES.get(roof.get("kernel"))
        line = {
            "metric": "qqmm FP4 TFLOP/s (% dense FP4 peak); quantize & qmv GB/s (% HBM peak)",
            "value": head["value"] * world, "unit": head["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 codes, e4m3 block scales, fp32 accumulate), bf16 io",
            "data": "synthetic (seeded torch generators; shapes and distributions of the workload configs)",
            "config": {"workload": f"{head_row}: " + {
                "prefill": "nvfp4 qqmm op, x [4096,4096] bf16 N(0,1), W [4096,4096] bf16 N(0,0.02) with 1% x50 "
                           "outliers, g = amax, SWIZZLED scales, y bf16",
                "gemv": "nvfp4 qmv, x [1,4096] bf16, W [14336,4096] pre-quantized"}.get(head_row, head_row),
                "rows_per_step": [r.name for r in rows], "l2": "flushed before every row: 256 MiB write, then 256 MiB read",
                "timing": "each row's ABI calls replayed as one CUDA graph per step; device time from events "
                          "recorded inside the graph before and after every call; each row's roofline kernel "
                          "also launched back to back over operand copies larger than L2, events around the "
                          "launches (roofline achieved; achieved_isolated is the flushed single call)",
                "parallelism": f"{world} ranks, each its own draw of every workload (no collective)" if world > 1
                               else "1 GPU"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": sum(r.launches + r.b2b_n * r.b2b_kernels for r in rows) * args.steps,
            "clocks": clocks,
            "rows": reports,
        }
        if unavailable:
            line["unavailable_rows"] = unavailable
        # last key, so that a tail of the line still shows it: the roofline
        # fractions of the three rows with stated targets (quantize and qmv
        # >= 0.70 of HBM, the large qqmm >= 0.60 of the dense FP4 peak), back
        # to back and as a flushed single call
        targets = {}
        for name, target in (("quant1g", 0.70), ("gemv", 0.70), ("gemv_chain", 0.70), ("prefill", 0.60)):
            rf = reports.get(name, {}).get("roofline")
            if rf:
                iso = rf.get("achieved_isolated", rf["achieved"]) / rf["peak"]
                targets[name] = {"kernel": rf.get("kernel"), "frac": round(rf["frac"], 4),
                                 "frac_isolated": round(iso, 4), "target": target}
        line["targets"] = targets
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the oracle (plain CPU code) on the same workload
# ---------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    d = workloads.make("prefill", device="cpu")
    for _ in range(args.warmup):  # untimed: the same step, its result discarded
        cpu_baseline_prefill(sample_rows=4, d=d)
    samples = [cpu_baseline_prefill(sample_rows=4, d=d) for _ in range(max(1, args.steps))]
    v = statistics.median(s["value"] for s in samples)
    ms_step = statistics.mean(s["seconds"] for s in samples) * 1e3
    line = {"impl": "reference", "metric": "qqmm FP4 TFLOP/s (% dense FP4 peak); quantize & qmv GB/s (% HBM peak)",
            "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 contraction of exactly decoded nvfp4 operands",
            "data": "synthetic (same seeded generators)",
            "config": {"workload": "prefill: nvfp4 qqmm op (oracle on a bounded sample of rows)"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "kind": "oracle", "cores": samples[0]["cores"],
                             "sample": samples[0]["sample"]},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--rows", nargs="*", default=None, help="subset of rows (default: all)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
