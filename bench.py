#!/usr/bin/env python3
"""Benchmark of the differential attention forward on B200.

One step = the whole hot path for one batch of the primary workload: the
per-head lambda kernel, then the prefill kernel (default workload: V2 causal
prefill, B2 Hq64 Hkv8 N8192 D128 bf16, layer 24).  The other workloads (V1
prefill with RMSNorm, both backwards, V2 64k decode contiguous and paged, a
serving-shaped paged decode, V1-layout 64k decode fused and unfused, the
low-rank forward and the SNR-vs-context-length sweep) are timed the same way
and reported, one compact row each, under "secondary" at the end of the line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl reference] [--no-cpu-baseline] [--no-secondary]

All inputs are synthetic (seeded, on the device), larger than L2, so no L2
flush is needed between timed steps.  Device times come from CUDA events on
the launching stream; for N > 1 (torchrun) each rank runs its own batch
(weak scaling, no collective on the data path) and rank 0 reports the max
time over ranks.
"""

from __future__ import annotations

import argparse
import functools
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import differential_attention_transformers_b200 as da  # noqa: E402
from differential_attention_transformers_b200 import inputs  # noqa: E402
from differential_attention_transformers_b200 import noise  # noqa: E402

METRIC = "diff-attn fwd prefill TFLOP/s & decode KV GB/s on 1 B200 (% of roofline)"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- work counts
def causal_pairs(Lq: int, Lk: int, causal: bool) -> int:
    """Number of (query, key) pairs a row-softmax sees (bottom-right causal mask)."""
    if not causal:
        return Lq * Lk
    off = Lk - Lq
    tot = 0
    # rows i see min(Lk, max(0, i + off + 1)) keys; sum in closed form by ranges
    lo = max(0, -off)                      # first row that sees >= 1 key
    hi = min(Lq, Lk - off)                 # rows [lo, hi) see i + off + 1 keys
    if hi > lo:
        tot += (hi - lo) * (off + 1) + (hi - 1 + lo) * (hi - lo) // 2
    if Lq > max(hi, lo):
        tot += (Lq - max(hi, lo)) * Lk     # rows that see every key
    return tot


def prefill_flops(w) -> int:
    """Executed-minimum FLOP: two QK^T and two PV products per diff head."""
    nc = causal_pairs(w.Lq, w.Lk, w.causal)
    if w.layout == "v2":
        return nc * 4 * w.d * w.H * w.B          # H = Q heads; each map 2d (QK) + 2dv (PV), dv == d
    return nc * (4 * w.d + 4 * w.dv) * w.H * w.B


def decode_bytes(w) -> int:
    """Algorithmic bytes of one decode step: the K and V caches read once."""
    per_key = (w.d + w.dv) * 2 if w.layout == "v2_decode" else (2 * w.d + w.dv) * 2
    return w.B * w.Hkv * w.Lk * per_key


# ----------------------------------------------------------------------------- peaks / clocks
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, read through NVML every few
    milliseconds on a background thread (reads only; no setting is touched).
    ``summary(t0, t1)`` summarises the samples taken between two host
    perf_counter() times, so a timed region of a few tens of milliseconds has
    a clock record of its own."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.dev, self.period = device_index, period_s
        self.samples, self.max_mhz, self.nv, self._stop = [], None, None, None

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
                h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = nv.nvmlDeviceGetHandleByIndex(self.dev)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
        except Exception:
            return self
        self.nv, self._stop = nv, threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.perf_counter(), mhz, [n for n, bit in bits if r & bit]))
                except Exception:
                    pass
                self._stop.wait(self.period)
        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join()
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self, t0=None, t1=None):
        sel = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(x[1] for x in sel), "sm_max_mhz": self.max_mhz,
                "reasons": sorted({n for x in sel for n in x[2]}), "samples": len(sel)}


# ----------------------------------------------------------------------------- workloads
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the current kernel on a smaller batch of the same workload;
# traffic grows with the batch (independent (batch, head) units), so a full
# launch is scaled by B / captured B.  None where no capture of the current
# kernel exists.
MEASURED_TRAFFIC = {
    "v2_prefill": (168.1e6 + 45.3e6, 1),       # prefill_kernel<128, PF_INFER>, B1
    "v1_prefill": (144.5e6 + 16.6e6, 2),       # prefill_kernel<64, PF_INFER>, B2, 4-row-block groups
    "v2_decode": (537.0e6 + 3.2e6, 2),         # decode_split_kernel<2, false>, B2
    "v2_decode_paged": (537.0e6 + 3.2e6, 2),   # decode_split_kernel<2, true>, B2, 16-token pages
}


def measured_traffic(name, B):
    t = MEASURED_TRAFFIC.get(name)
    return None if t is None else t[0] * B / t[1]


class Prefill:
    def __init__(self, w, device):
        self.w = w
        self.x = inputs.make(w, device=device)
        self.lp = inputs.lambda_params(w, device=device)
        self.init = da.lambda_init(w.layer)
        self.lam = torch.empty(w.pairs, dtype=torch.float32, device=device)
        out_h = w.pairs
        self.out = torch.empty((w.B, out_h, w.Lq, w.dv), dtype=w.dtype, device=device)
        self.launches_per_step = 2
        self.k_start = torch.cuda.Event(enable_timing=True)
        self.k_end = torch.cuda.Event(enable_timing=True)

    def step(self, ev=None):
        w, x = self.w, self.x
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        if ev is not None:
            ev[0].record()
        if w.layout == "v2":
            da.fwd_v2(x["q"], x["k"], x["v"], self.lam, causal=w.causal, out=self.out)
        else:
            da.fwd_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], self.lam, causal=w.causal,
                      rmsnorm=w.rmsnorm, eps=1e-5, out=self.out)
        if ev is not None:
            ev[1].record()

    def work(self):
        return prefill_flops(self.w) / 1e12, "TFLOP/s"

    def host_call(self, host):
        w = self.w
        lam = da.compute_lambda(*host["lp"], self.init)
        if w.layout == "v2":
            return da.fwd_v2(host["q"], host["k"], host["v"], lam, causal=w.causal)
        return da.fwd_v1(host["q1"], host["k1"], host["q2"], host["k2"], host["v"], lam, causal=w.causal,
                         rmsnorm=w.rmsnorm, eps=1e-5)


class Decode:
    def __init__(self, w, device, fused=True):
        self.w = w
        self.fused = fused
        self.x = inputs.make(w, device=device)
        self.lp = inputs.lambda_params(w, device=device)
        self.init = da.lambda_init(w.layer)
        self.lam = torch.empty(w.pairs, dtype=torch.float32, device=device)
        self.out = torch.empty((w.B, w.pairs, w.dv), dtype=w.dtype, device=device)
        self.ws = torch.empty(da.decode_workspace_size(w.B, w.Hkv, w.Lk, w.dv), dtype=torch.uint8, device=device)
        passes = 1 if (w.layout == "v2_decode" or fused) else 2
        self.launches_per_step = 2 + passes

    def step(self, ev=None):
        w, x = self.w, self.x
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        if ev is not None:
            ev[0].record()
        if w.layout == "v2_decode":
            da.decode_v2(x["q"], x["k"], x["v"], self.lam, out=self.out, workspace=self.ws)
        else:
            da.decode_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], self.lam, fused=self.fused, out=self.out,
                         workspace=self.ws)
        if ev is not None:
            ev[1].record()

    def work(self):
        b = decode_bytes(self.w)
        if self.w.layout == "v1_decode" and not self.fused:
            b += self.w.B * self.w.Hkv * self.w.Lk * self.w.dv * 2   # V read a second time
        return b / 1e9, "GB/s"

    def host_call(self, host):
        w = self.w
        lam = da.compute_lambda(*host["lp"], self.init)
        if w.layout == "v2_decode":
            return da.decode_v2(host["q"], host["k"], host["v"], lam)
        return da.decode_v1(host["q1"], host["k1"], host["q2"], host["k2"], host["v"], lam, fused=self.fused)


PAGE_SIZE = 16   # paged decode secondary: 16-token pages


class PagedDecode:
    """The V2 decode workload with its caches in a shuffled pool of 16-token pages."""

    def __init__(self, w, device):
        self.w = w
        x = inputs.make(w, device=device)
        kp, vp, bt, sl = inputs.paged_cache(x["k"], x["v"], PAGE_SIZE, seed=w.seed)
        del x["k"], x["v"]
        self.x = {"q": x["q"], "k_pages": kp, "v_pages": vp, "block_table": bt, "seq_lens": sl}
        self.lp = inputs.lambda_params(w, device=device)
        self.init = da.lambda_init(w.layer)
        self.lam = torch.empty(w.pairs, dtype=torch.float32, device=device)
        self.out = torch.empty((w.B, w.pairs, w.dv), dtype=w.dtype, device=device)
        self.ws = torch.empty(da.decode_paged_workspace_size(w.B, w.Hkv), dtype=torch.uint8, device=device)
        self.launches_per_step = 3

    def step(self, ev=None):
        x = self.x
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        if ev is not None:
            ev[0].record()
        da.decode_v2_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], self.lam,
                           out=self.out, workspace=self.ws)
        if ev is not None:
            ev[1].record()

    def work(self):
        return decode_bytes(self.w) / 1e9, "GB/s"

    def host_call(self, host):
        lam = da.compute_lambda(*host["lp"], self.init)
        return da.decode_v2_paged(host["q"], host["k_pages"], host["v_pages"], host["block_table"],
                                  host["seq_lens"], lam)


class ServingDecode:
    """A serving-shaped paged V2 decode: 256 sequences of mixed lengths
    (16..4096 tokens) in a shared pool of 16-token pages, one query token each."""

    def __init__(self, device, shape=None):
        self.shape = dict(inputs.SERVING_SHAPE if shape is None else shape)
        sh = self.shape
        self.x = inputs.serving_cache(**sh, device=device)
        self.tokens = int(self.x["seq_lens"].sum())
        gen = torch.Generator(device=device).manual_seed(1014)
        self.lp = tuple(torch.randn(sh["Hq"] // 2, 128, generator=gen, device=device) * 0.1 for _ in range(4))
        self.init = da.lambda_init(24)
        self.lam = torch.empty(sh["Hq"] // 2, dtype=torch.float32, device=device)
        self.out = torch.empty((sh["B"], sh["Hq"] // 2, 128), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(da.decode_paged_workspace_size(sh["B"], sh["Hkv"]), dtype=torch.uint8, device=device)
        self.launches_per_step = 3

    def step(self, ev=None):
        x = self.x
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        if ev is not None:
            ev[0].record()
        da.decode_v2_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["seq_lens"], self.lam,
                           out=self.out, workspace=self.ws)
        if ev is not None:
            ev[1].record()

    def work(self):
        """Bytes of the K and V tokens the sequences hold, each read once."""
        return self.tokens * self.shape["Hkv"] * (128 + 128) * 2 / 1e9, "GB/s"

    host_path = "the serving-shaped decode is timed on device tensors only"


def backward_flops(w) -> float:
    """Executed-minimum FLOP of the backward: five contractions per map and
    visible (row, key) pair -- S (2d), dP (2dv), dV (2dv), dQ (2d), dK (2d) --
    against the forward's two (2d + 2dv); 2.5 x the forward for V2."""
    return prefill_flops(w) * (6 * w.d + 4 * w.dv) / (2 * w.d + 2 * w.dv)


class Backward:
    """Backward of a prefill workload: the training forward runs once (untimed)
    for its statistics, then each step is lambda + the full backward."""

    def __init__(self, w, device):
        self.w = w
        self.x = inputs.make(w, device=device)
        self.lp = inputs.lambda_params(w, device=device)
        self.init = da.lambda_init(w.layer)
        self.lam = torch.empty(w.pairs, dtype=torch.float32, device=device)
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        gen = torch.Generator(device=device).manual_seed(w.seed + 1)
        self.dout = torch.randn((w.B, w.pairs, w.Lq, w.dv), generator=gen, device=device).to(w.dtype)
        x = self.x
        if w.layout == "v2":
            _, self.lse, self.om = da.fwd_v2_train(x["q"], x["k"], x["v"], self.lam, causal=w.causal)
            nws = da.load().diffattn_bwd_v2_workspace_size(w.B, w.H, w.Lq)
            self.launches_per_step = 6   # lambda, prep, dlambda, dQ, dK/dV, lambda's parameter gradients
        else:
            self.out, self.lse, self.om, self.rstd, self.o2c = da.fwd_v1_train(x["q1"], x["k1"], x["q2"], x["k2"], x["v"],
                                                                     self.lam, causal=w.causal, rmsnorm=w.rmsnorm)
            nws = da.load().diffattn_bwd_v1_workspace_size(w.B, w.H, w.Hkv, w.Lq, w.Lk, int(w.rmsnorm))
            # lambda, [RMSNorm gradient], prep, dlambda, dQ, dK/dV, lambda's parameter gradients
            self.launches_per_step = 7 if w.rmsnorm else 6
        self.ws = torch.empty(int(nws), dtype=torch.uint8, device=device)

    def step(self, ev=None):
        w, x = self.w, self.x
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        if ev is not None:
            ev[0].record()
        if w.layout == "v2":
            dlam = da.bwd_v2(x["q"], x["k"], x["v"], self.lam, self.dout, self.lse, self.om, causal=w.causal,
                             workspace=self.ws)[-1]
        else:
            dlam = da.bwd_v1(x["q1"], x["k1"], x["q2"], x["k2"], x["v"], self.lam, self.dout, self.out, self.lse,
                             self.om, self.rstd, self.o2c, causal=w.causal, rmsnorm=w.rmsnorm,
                             workspace=self.ws)[-1]
        da.lambda_backward(*self.lp, dlam)
        if ev is not None:
            ev[1].record()

    def work(self):
        return backward_flops(self.w) / 1e12, "TFLOP/s"

    host_path = "the backward is timed on device tensors only"


def sweep_bytes(n=inputs.SWEEP_INSTANCES, lengths=inputs.SWEEP_LENGTHS) -> int:
    """Algorithmic bytes of one sweep step: every context length decoded twice
    (plain and difference), each reading K1, K2 (64 wide) and V (128 wide) once."""
    return sum(2 * n * N * (64 + 64 + 128) * 2 for N in lengths)


class SnrSweep:
    """The SNR-vs-context-length sweep (tutorial exercise 1): one step decodes
    the noise construction at every length from 1k to 256k keys, with lambda = 0
    (plain softmax) and lambda = 0.5 (the difference), on the V1 decode kernel."""

    def __init__(self, device, n=inputs.SWEEP_INSTANCES, lengths=inputs.SWEEP_LENGTHS):
        self.n, self.lengths = n, tuple(lengths)
        base = inputs.noise_sweep(n, max(self.lengths), device=device)
        self.parts = [inputs.sweep_prefix(base, N) for N in self.lengths]
        del base
        self.lams = (torch.zeros(1, dtype=torch.float32, device=device),
                     torch.full((1,), 0.5, dtype=torch.float32, device=device))
        self.outs = [[torch.empty((n, 1, 128), dtype=torch.bfloat16, device=device) for _ in self.lams]
                     for _ in self.lengths]
        self.ws = torch.empty(da.decode_workspace_size(n, 1, max(self.lengths)), dtype=torch.uint8, device=device)
        self.launches_per_step = 2 * len(self.lengths) * 2   # split-KV kernel + combine, per decode

    def step(self, ev=None):
        if ev is not None:
            ev[0].record()
        for p, outs in zip(self.parts, self.outs):
            for lam, out in zip(self.lams, outs):
                da.decode_v1(p["q1"], p["k1"], p["q2"], p["k2"], p["v"], lam, out=out, workspace=self.ws)
        if ev is not None:
            ev[1].record()

    def work(self):
        return sweep_bytes(self.n, self.lengths) / 1e9, "GB/s"

    def summary(self):
        return [noise.summarize(N, o[0][:, 0, 0].float(), o[0][:, 0, 1].float(), o[1][:, 0, 0].float(),
                                o[1][:, 0, 1].float()) for N, o in zip(self.lengths, self.outs)]

    def compact_summary(self):
        """Medians per context length: [N, SNR plain, SNR difference, plain noise fraction]."""
        return [[r["N"], float(f"{r['snr_plain'][1]:.3g}"), float(f"{r['snr_diff'][1]:.3g}"),
                 float(f"{r['noise_fraction_plain'][1]:.3g}")] for r in self.summary()]

    host_path = "the sweep is timed on device tensors only"


def lowrank_flops(B, H, L, **_) -> float:
    """Executed-min FLOP of the low-rank forward's attention: one QK^T and one
    PV product per head over the causal pairs (the scan of N V adds about
    6 r dv FLOP per row and key-step, under 1 % here, and is not counted)."""
    nc = causal_pairs(L, L, True)
    return nc * (2 * 128 + 2 * 128) * H * B


class LowRank:
    """The fixed low-rank substitute for A2: one step is lambda, then
    out = A1 V - lambda N V (single-map prefill, then the N V scan)."""

    def __init__(self, device, shape=None):
        self.shape = dict(inputs.LOWRANK_SHAPE if shape is None else shape)
        sh = self.shape
        self.x = inputs.lowrank_inputs(**sh, device=device)
        gen = torch.Generator(device=device).manual_seed(1012)
        self.lp = tuple(torch.randn(sh["H"], 128, generator=gen, device=device) * 0.1 for _ in range(4))
        self.init = da.lambda_init(24)
        self.lam = torch.empty(sh["H"], dtype=torch.float32, device=device)
        self.out = torch.empty((sh["B"], sh["H"], sh["L"], 128), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(int(da.load().diffattn_fwd_lowrank_workspace_size(sh["B"], sh["H"], sh["L"], sh["L"],
                                                                                sh["r"], 1)),
                              dtype=torch.uint8, device=device)
        self.launches_per_step = 5   # lambda, single-map prefill, chunk sums, prefix, emit

    def step(self, ev=None):
        x = self.x
        da.compute_lambda(*self.lp, self.init, out=self.lam)
        if ev is not None:
            ev[0].record()
        da.fwd_lowrank(x["q"], x["k"], x["v"], x["F"], x["G"], self.lam, causal=True, out=self.out,
                       workspace=self.ws)
        if ev is not None:
            ev[1].record()

    def work(self):
        return lowrank_flops(**self.shape) / 1e12, "TFLOP/s"

    host_path = "the low-rank forward is timed on device tensors only"


def workload_work(name):
    """(algorithmic work of one step, unit) of a bench workload."""
    if name == "v2_decode_serving":
        return None, "GB/s"     # set by the drawn lengths (ServingDecode.work)
    if name == "snr_sweep":
        return sweep_bytes() / 1e9, "GB/s"
    if name == "lowrank_prefill":
        return lowrank_flops(**inputs.LOWRANK_SHAPE) / 1e12, "TFLOP/s"
    w = inputs.WORKLOADS[base_workload(name)]
    if name.endswith("_backward"):
        return backward_flops(w) / 1e12, "TFLOP/s"
    if w.layout in ("v1", "v2"):
        return prefill_flops(w) / 1e12, "TFLOP/s"
    return decode_bytes(w) / 1e9 * (1.5 if name.endswith("_unfused") else 1.0), "GB/s"


def base_workload(name):
    """The workload a bench name is built on (variants share their base's shapes)."""
    return {"v2_backward": "v2_prefill", "v1_backward": "v1_prefill", "v2_decode_paged": "v2_decode",
            "v1_decode_unfused": "v1_decode"}.get(name, name)


def make_runner(name, device):
    if name == "v2_decode_serving":
        return ServingDecode(device)
    if name == "snr_sweep":
        return SnrSweep(device)
    if name == "lowrank_prefill":
        return LowRank(device)
    if name.endswith("_backward"):
        return Backward(inputs.WORKLOADS[base_workload(name)], device)
    if name == "v2_decode_paged":
        return PagedDecode(inputs.WORKLOADS["v2_decode"], device)
    w = inputs.WORKLOADS[name.replace("_unfused", "")]
    if w.layout in ("v1", "v2"):
        return Prefill(w, device)
    return Decode(w, device, fused=not name.endswith("_unfused"))


def describe(name):
    if name == "v2_decode_serving":
        sh = inputs.SERVING_SHAPE
        return {"workload": name, "layout": "v2_decode", "B": sh["B"], "heads": sh["Hq"], "kv_heads": sh["Hkv"],
                "Lq": 1, "Lk": f"uniform {sh['min_len']}..{sh['max_len']}", "d": 128, "dv": 128, "layer": 24,
                "mode": f"paged: shuffled pool of {sh['page_size']}-token pages, mixed lengths",
                "l2": "caches larger than L2 (126 MB): no flush between steps"}
    if name == "lowrank_prefill":
        sh = inputs.LOWRANK_SHAPE
        return {"workload": name, "layout": "one Q head per output head", "B": sh["B"], "heads": sh["H"],
                "kv_heads": sh["Hkv"], "Lq": sh["L"], "Lk": sh["L"], "d": 128, "dv": 128, "causal": True,
                "rank": sh["r"], "layer": 24,
                "mode": "A1 V - lambda N V, N fixed from positional factors F, G ~ U(0,1)",
                "l2": "inputs larger than L2 (126 MB): no flush between steps"}
    if name == "snr_sweep":
        return {"workload": name, "layout": "v1_decode", "instances": inputs.SWEEP_INSTANCES,
                "Lk": list(inputs.SWEEP_LENGTHS), "d": 64, "dv": 128, "lambda": [0.0, 0.5],
                "mode": "noise construction (key 0 = 5q among N(0,1) keys), plain and difference rows; "
                        "V = two indicator columns",
                "l2": "inputs larger than L2 (126 MB) at the long lengths; no flush between steps"}
    w = inputs.WORKLOADS[base_workload(name)]
    d = {"workload": name, "layout": w.layout, "B": w.B, "heads": w.H, "kv_heads": w.Hkv, "Lq": w.Lq, "Lk": w.Lk,
         "d": w.d, "dv": w.dv, "causal": w.causal, "layer": w.layer, "rmsnorm": w.rmsnorm,
         "l2": "inputs larger than L2 (126 MB): no flush between steps"}
    if name.endswith("_unfused"):
        d["mode"] = "two passes, V read twice (comparison)"
    if name == "v2_backward":
        d["mode"] = "backward: dQ, dK, dV, dlambda from the training forward's statistics; dO ~ N(0,1)"
    if name == "v1_backward":
        d["mode"] = ("backward: dQ1, dK1, dQ2, dK2, dV, dlambda (RMSNorm gradient first) from the training "
                     "forward's statistics; dO ~ N(0,1)")
    if name.endswith("_paged"):
        d["mode"] = f"paged: shuffled pool of {PAGE_SIZE}-token pages [num_pages, {PAGE_SIZE}, Hkv, 128], block table"
    return d


# ----------------------------------------------------------------------------- timing
def time_runner(r, steps, warmup, dist_on, window=None):
    """W untimed steps, then K steps bracketed by a barrier and a synchronize
    on both sides; CUDA events on the launching stream give the whole region
    and each step's dominant launch.  ``window``, a list, receives the host
    perf_counter() times around the timed region (for the clock record)."""
    for _ in range(warmup):
        r.step()
    torch.cuda.synchronize()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record()
    for i in range(steps):
        r.step(kev[i])
    end.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if dist_on:
        torch.distributed.barrier()
    if window is not None:
        window[:] = [t0, t1]
    total_ms = start.elapsed_time(end)
    kern_ms = sum(a.elapsed_time(b) for a, b in kev) / steps
    return total_ms, kern_ms


def keep_busy(r, seconds):
    """Run untimed steps for about `seconds` (device time)."""
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        for _ in range(8):
            r.step()
        torch.cuda.synchronize()


def max_over_ranks(x, dist_on):
    """Max of a per-rank time over all ranks (the slowest rank sets the step time)."""
    if not dist_on:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(work_per_rank, world, ms_per_step):
    """Whole-job throughput: every rank processes its own batch (weak scaling)."""
    return work_per_rank * world / (ms_per_step / 1e3)


def e2e_measure(r, steps):
    """Same metric through the public API with pinned HOST buffers: the
    host->device copies of the step's inputs and the device->host copy of its
    output are inside the timed region.  A runner without a host path names
    why in its ``host_path`` string."""
    if isinstance(getattr(r, "host_path", None), str):
        raise NotImplementedError(r.host_path)
    host = {k: v.cpu().pin_memory() for k, v in r.x.items()}
    host["lp"] = [t.cpu().pin_memory() for t in r.lp]
    h2d = sum(v.numel() * v.element_size() for k, v in host.items() if k != "lp")
    h2d += sum(t.numel() * t.element_size() for t in host["lp"])
    # Two warm-up calls: a call's pinned result buffer is reused from torch's
    # host cache once an earlier one has been released, but the first timed
    # call would otherwise allocate it afresh (a one-time cost of tens of ms).
    out = r.host_call(host)
    out = r.host_call(host)
    d2h = out.numel() * out.element_size()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    s.record()
    for _ in range(steps):
        out = None                               # the previous result goes back to the cache first
        out = r.host_call(host)
    e.record()
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) * 1e3 / steps
    dev_ms = s.elapsed_time(e) / steps
    ms = max(wall, dev_ms)
    work, unit = r.work()
    del host
    h2d_gbs, d2h_gbs = pinned_copy_gbs()
    # the copies alone, at the measured pinned bandwidths, in sequence: a floor
    # for the step when the kernel is fully hidden behind them
    copy_ms = (h2d / (h2d_gbs * 1e9) + d2h / (d2h_gbs * 1e9)) * 1e3 if h2d_gbs and d2h_gbs else None
    return {"value": work / (ms / 1e3), "unit": unit, "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pinned_h2d_gbs": h2d_gbs, "pinned_d2h_gbs": d2h_gbs, "copy_floor_ms": copy_ms}


def pinned_copy_gbs(nbytes=256 << 20, reps=5):
    """Measured host<->device bandwidth of one large pinned copy each way
    (GB/s, best of a few), the ceiling the end-to-end number is held to."""
    try:
        host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        dev = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        out = []
        for src, dst in ((host, dev), (dev, host)):
            best = None
            for _ in range(reps):
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record()
                dst.copy_(src, non_blocking=True)
                e.record()
                torch.cuda.synchronize()
                ms = s.elapsed_time(e)
                best = ms if best is None else min(best, ms)
            out.append(nbytes / (best / 1e3) / 1e9 if best else None)
        del host, dev
        return tuple(out)
    except Exception:
        return None, None


SPEC_HBM_GBS = 8000.0   # the HBM3e figure the decode target is stated against (~8 TB/s)


def roofline(r, kern_ms, peaks, power_capped=False, name=None):
    """Achieved work rate of the step's dominant kernel against the measured peak.

    A tensor-bound kernel is compared with the measured burst cuBLAS bf16
    figure: each prefill launch lasts a few milliseconds and is timed on its
    own, which is the burst regime (a power cap seen on the clocks is a note,
    not another roofline).  The fraction of the sustained figure is kept as a
    side field.  An HBM-bound kernel is compared with the measured copy
    bandwidth; a read-only stream can run above a read+write copy, so the
    fraction of the ~8 TB/s HBM3e figure is given beside it.  traffic: the
    DRAM bytes of one launch from the kernel's ncu capture, scaled to this
    batch (None without a capture of the current kernel)."""
    work, unit = r.work()
    w = getattr(r, "w", None)
    traffic = measured_traffic(name, w.B) if (name is not None and w is not None) else None
    ach = work / (kern_ms / 1e3)
    if unit == "TFLOP/s":
        peak = peaks["bf16_tflops"]
        out = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
               "traffic": traffic, "peak_kind": f"{peaks['source']} burst cuBLAS bf16", "kernel_ms": kern_ms}
        if peaks.get("bf16_tflops_sustained"):
            out["frac_of_sustained"] = ach / peaks["bf16_tflops_sustained"]
        if power_capped:
            out["note"] = "sw_power_cap seen during the timed region"
        return out
    peak = peaks["hbm_gbs"]
    out = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak, "traffic": traffic,
           "peak_kind": f"{peaks['source']} HBM copy (read+write)", "frac_of_8tbs": ach / SPEC_HBM_GBS,
           "kernel_ms": kern_ms}
    if ach > peak:
        out["note"] = "read-only stream above the read+write copy figure"
    return out


def compact(name, r, total_ms, kern_ms, steps, rf):
    """One secondary row: [value, unit, ms_per_step, kernel_ms, frac, frac_of_8tbs or None]."""
    work, unit = r.work()
    ms = total_ms / steps
    return [round(work / (ms / 1e3), 2), unit, round(ms, 4), round(kern_ms, 4), round(rf["frac"], 4),
            round(rf["frac_of_8tbs"], 4) if "frac_of_8tbs" in rf else None]


SECONDARY_COLS = ["value", "unit", "ms_per_step", "kernel_ms", "frac", "frac_of_8tbs", "sm_mhz"]

# Idle time before each secondary row's warm-up, so that its timed region
# starts from the regime of the headline one (a launch timed on its own, the
# burst clock) rather than from the power-capped clock the rows before it left.
SETTLE_S = 1.0


# ----------------------------------------------------------------------------- CPU oracle arm
def cpu_oracle_lowrank(cores, budget_s):
    """The oracle's low-rank head on whole (batch, head) slices of the workload."""
    from oracle import lowrank as olr
    sh = inputs.LOWRANK_SHAPE
    x = _lowrank_host_inputs()
    grp = sh["H"] // sh["Hkv"]
    per_slice = lowrank_flops(**sh) / (sh["B"] * sh["H"]) / 1e12
    done, t_total, n = 0.0, 0.0, 0
    for h in range(sh["H"]):
        for b in range(sh["B"]):
            t0 = time.perf_counter()
            olr.lowrank_head(x["q"][b, h], x["k"][b, h // grp], x["v"][b, h // grp], x["F"][h].numpy(),
                             x["G"][h].numpy(), 0.5, True)
            t_total += time.perf_counter() - t0
            done += per_slice
            n += 1
            if t_total >= budget_s:
                break
        if t_total >= budget_s:
            break
    return {"value": done / t_total, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of {sh['B'] * sh['H']} (batch, head) slices, all {sh['L']} rows, fp64 NumPy",
            "seconds": t_total}


@functools.lru_cache(maxsize=1)
def _lowrank_host_inputs():
    return inputs.lowrank_inputs(**inputs.LOWRANK_SHAPE)


@functools.lru_cache(maxsize=1)
def _sweep_host_inputs():
    """The sweep's inputs on the host, drawn once per process (about 12 s)."""
    return inputs.noise_sweep(inputs.SWEEP_INSTANCES, inputs.SWEEP_LENGTHS[-1])


def cpu_oracle_sweep(cores, budget_s):
    """The oracle's noise probe on instances of the sweep, longest context
    first, both rows (plain and difference) per probe; bytes counted as on the
    GPU (K1, K2 and V of the instance, per row)."""
    from oracle import diffattn as orc
    N = inputs.SWEEP_LENGTHS[-1]
    x = _sweep_host_inputs()
    done, t_total, n = 0.0, 0.0, 0
    for i in range(inputs.SWEEP_INSTANCES):
        t0 = time.perf_counter()
        orc.noise_probe(x["q1"][i:i + 1, 0], x["k1"][i:i + 1, 0], x["q2"][i:i + 1, 0], x["k2"][i:i + 1, 0], 0.5)
        t_total += time.perf_counter() - t0
        done += 2 * N * (64 + 64 + 128) * 2 / 1e9
        n += 1
        if t_total >= budget_s:
            break
    return {"value": done / t_total, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of {inputs.SWEEP_INSTANCES} instances at {N} keys, plain and difference rows, fp64 NumPy",
            "seconds": t_total}


@functools.lru_cache(maxsize=1)
def _serving_host_inputs():
    return inputs.serving_cache(**inputs.SERVING_SHAPE)


def cpu_oracle_serving(cores, budget_s):
    """The oracle's paged decode on whole sequences of the serving batch, in
    order; bytes counted as on the GPU (the sequence's K and V tokens)."""
    import numpy as np
    from oracle import diffattn as orc
    x = _serving_host_inputs()
    sh = inputs.SERVING_SHAPE
    lam = np.full(sh["Hq"] // 2, 0.5)
    done, t_total, n = 0.0, 0.0, 0
    for b in range(sh["B"]):
        t0 = time.perf_counter()
        orc.decode_v2_paged(x["q"][b:b + 1], x["k_pages"], x["v_pages"], x["block_table"][b:b + 1],
                            x["seq_lens"][b:b + 1], lam)
        t_total += time.perf_counter() - t0
        done += int(x["seq_lens"][b]) * sh["Hkv"] * 256 * 2 / 1e9
        n += 1
        if t_total >= budget_s:
            break
    return {"value": done / t_total, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of {sh['B']} sequences in order, fp64 NumPy", "seconds": t_total}


def cpu_oracle_run(name, budget_s=12.0):
    """Time the fp64 oracle, as it stands, on a bounded sample of the workload.

    Prefill: whole (batch, head) slices over all rows; decode: whole (batch,
    KV head) groups.  The work done is counted with the same convention as
    the GPU metric and divided by the measured time."""
    import numpy as np
    from oracle import diffattn as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        cores = len(os.sched_getaffinity(0))
    if name == "snr_sweep":
        return cpu_oracle_sweep(cores, budget_s)
    if name == "v2_decode_serving":
        return cpu_oracle_serving(cores, budget_s)
    if name == "lowrank_prefill":
        return cpu_oracle_lowrank(cores, budget_s)
    paged, backward = name == "v2_decode_paged", name.endswith("_backward")
    w = inputs.WORKLOADS[base_workload(name)]
    x = inputs.make(w, device="cpu") if w.layout in ("v1", "v2") else None
    lam = np.full(w.pairs, 0.5)
    done_work, t_total, n = 0.0, 0.0, 0
    if w.layout in ("v1", "v2"):
        per_slice = (backward_flops(w) if backward else prefill_flops(w)) / (w.B * w.pairs) / 1e12
        units = [(b, h) for h in range(w.pairs) for b in range(w.B)]
        if backward:
            from oracle import backward as obwd
            dout = torch.randn((1, w.Lq, w.dv), generator=torch.Generator().manual_seed(w.seed)).to(w.dtype)
        for b, h in units:
            t0 = time.perf_counter()
            if backward and w.layout == "v1":
                g = h // (w.H // w.Hkv)
                obwd.head_backward(x["q1"][b, h], x["k1"][b, g], x["q2"][b, h], x["k2"][b, g], x["v"][b, g], lam[h],
                                   dout[0], causal=w.causal, rms=w.rmsnorm)
            elif backward:
                g = (2 * h) // (w.H // w.Hkv)
                obwd.head_backward(x["q"][b, 2 * h], x["k"][b, g], x["q"][b, 2 * h + 1], x["k"][b, g], x["v"][b, g],
                                   lam[h], dout[0], causal=w.causal)
            elif w.layout == "v2":
                g = (2 * h) // (w.H // w.Hkv)
                orc.diffattn_v2(x["q"][b:b + 1, 2 * h:2 * h + 2], x["k"][b:b + 1, g:g + 1],
                                x["v"][b:b + 1, g:g + 1], lam[h:h + 1], causal=w.causal)
            else:
                g = h // (w.H // w.Hkv)
                s = lambda t, hh: t[b:b + 1, hh:hh + 1]  # noqa: E731
                orc.diffattn_v1(s(x["q1"], h), s(x["k1"], g), s(x["q2"], h), s(x["k2"], g), s(x["v"], g),
                                lam[h:h + 1], causal=w.causal, rms=w.rmsnorm)
            t_total += time.perf_counter() - t0
            done_work += per_slice
            n += 1
            if t_total >= budget_s:
                break
        unit = "TFLOP/s"
        sample = f"{n} of {w.B * w.pairs} (batch, head) slices, all {w.Lq} rows, fp64 NumPy"
    else:
        gen = torch.Generator().manual_seed(w.seed)
        grp = w.H // w.Hkv
        per_group = decode_bytes(w) / (w.B * w.Hkv) / 1e9
        for b in range(w.B):
            for g in range(w.Hkv):
                if w.layout == "v2_decode":
                    q = (torch.randn(1, grp, w.d, generator=gen) * w.std).to(torch.bfloat16)
                    kc = (torch.randn(1, 1, w.Lk, w.d, generator=gen) * w.std).to(torch.bfloat16)
                    vc = (torch.randn(1, 1, w.Lk, w.dv, generator=gen) * w.std).to(torch.bfloat16)
                    if paged:
                        kp, vp, bt, sl = inputs.paged_cache(kc, vc, PAGE_SIZE, seed=b * w.Hkv + g)
                        t0 = time.perf_counter()
                        orc.decode_v2_paged(q, kp, vp, bt, sl, lam[: grp // 2])
                    else:
                        t0 = time.perf_counter()
                        orc.decode_v2(q, kc, vc, lam[: grp // 2])
                else:
                    q1 = (torch.randn(1, grp, w.d, generator=gen) * w.std).to(torch.bfloat16)
                    k1 = (torch.randn(1, 1, w.Lk, w.d, generator=gen) * w.std).to(torch.bfloat16)
                    vc = (torch.randn(1, 1, w.Lk, w.dv, generator=gen) * w.std).to(torch.bfloat16)
                    t0 = time.perf_counter()
                    orc.decode_v1(q1, k1, q1, k1, vc, lam[:grp])
                t_total += time.perf_counter() - t0
                done_work += per_group
                n += 1
                if t_total >= budget_s:
                    break
            if t_total >= budget_s:
                break
        unit = "GB/s"
        sample = f"{n} of {w.B * w.Hkv} (batch, KV head) groups, full cache, fp64 NumPy"
    return {"value": done_work / t_total, "unit": unit, "cores": int(cores), "kind": "oracle", "sample": sample,
            "seconds": t_total}


def _rounded(x, digits=6):
    """Floats to `digits` significant digits (keeps the JSON line short)."""
    if isinstance(x, float):
        return float(f"{x:.{digits}g}")
    if isinstance(x, dict):
        return {k: _rounded(v, digits) for k, v in x.items()}
    if isinstance(x, list):
        return [_rounded(v, digits) for v in x]
    return x


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="v2_prefill",
                    choices=["v2_prefill", "v1_prefill", "v2_backward", "v1_backward", "v2_decode", "v2_decode_paged",
                             "v2_decode_serving", "v1_decode", "v1_decode_unfused", "snr_sweep", "lowrank_prefill"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch size of the workload (smaller profiling cases)")
    args = ap.parse_args()
    if args.batch is not None and args.workload not in ("snr_sweep", "lowrank_prefill", "v2_decode_serving"):
        base = base_workload(args.workload)
        inputs.WORKLOADS[base] = inputs.with_shape(inputs.WORKLOADS[base], B=args.batch)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # The reference arm is the fp64 CPU oracle, on rank 0 only.
        if rank != 0:
            return 0
        steps = max(1, args.steps)
        res = [cpu_oracle_run(args.workload, budget_s=max(2.0, 60.0 / (steps + args.warmup)))
               for _ in range(steps + max(0, args.warmup))][args.warmup:] or [None]
        vals = [r["value"] for r in res]
        v = statistics.median(vals)
        cb = dict(res[-1])
        cb["value"] = v
        unit = cb["unit"]
        # One step is one bounded sample of the workload: ms_per_step is its
        # measured duration; the time the whole workload would take at this
        # rate is extrapolated and labelled so.
        ms_step = statistics.mean(r["seconds"] for r in res) * 1e3
        work_unit = workload_work(args.workload)[0]
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus,
                "steps": steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": dict(describe(args.workload), parallelism="single GPU"),
                "cpu_baseline": cb,
                "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "step": "one bounded sample of the workload per step (see cpu_baseline.sample)"}
        if work_unit:
            line["full_workload_ms_extrapolated"] = work_unit / v * 1e3
        print(json.dumps(line))
        return 0

    dist_on = world > 1
    if dist_on:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    peaks = measured_peaks()

    r = make_runner(args.workload, device)
    win, win_s = [], []
    with ClockSampler(torch.cuda.current_device()) as clk:
        # The headline region starts from the warm-up alone: a few tens of
        # milliseconds, the regime of a launch timed on its own (burst).
        total_ms, kern_ms = time_runner(r, args.steps, args.warmup, dist_on, win)
        # Then the same steps after a second of continuous load, where a
        # power cap may hold the clock lower (sustained), reported beside it.
        keep_busy(r, 1.0)
        sus_total, sus_kern = time_runner(r, args.steps, 0, dist_on, win_s)
    total_ms = max_over_ranks(total_ms, dist_on)
    sus_total = max_over_ranks(sus_total, dist_on)
    ms = total_ms / args.steps
    work, unit = r.work()
    value = aggregate(work, world, ms)
    clocks = clk.summary(*win) if win else clk.summary()
    clocks_s = clk.summary(*win_s) if win_s else clk.summary()
    capped = "sw_power_cap" in clocks["reasons"]
    rf = roofline(r, kern_ms, peaks, capped, args.workload)
    rf_s = roofline(r, sus_kern, peaks, "sw_power_cap" in clocks_s["reasons"], args.workload)
    sustained = {"value": aggregate(work, world, sus_total / args.steps), "ms_per_step": sus_total / args.steps,
                 "kernel_ms": sus_kern, "frac": rf_s.get("frac_of_sustained", rf_s["frac"]),
                 "sm_mhz": clocks_s["sm_mhz"], "reasons": clocks_s["reasons"]}

    secondary, snr = {}, None
    if isinstance(r, SnrSweep):
        snr = r.compact_summary()
    if not args.no_secondary and rank == 0 and not dist_on:
        names = ["v1_prefill", "v2_backward", "v1_backward", "v2_decode", "v2_decode_paged", "v2_decode_serving",
                 "v1_decode", "v1_decode_unfused", "lowrank_prefill", "snr_sweep", "v2_prefill"]
        n2 = max(3, args.steps // 2)
        with ClockSampler(torch.cuda.current_device()) as clk2:
            for name in names:
                if name == args.workload:
                    continue
                r2 = make_runner(name, device)
                torch.cuda.synchronize()
                time.sleep(SETTLE_S)
                w2 = []
                t2, k2 = time_runner(r2, n2, args.warmup, False, w2)
                c2 = clk2.summary(*w2)
                rf2 = roofline(r2, k2, peaks, "sw_power_cap" in c2["reasons"], name)
                mhz = c2["sm_mhz"]
                secondary[name] = compact(name, r2, t2, k2, n2, rf2) + [None if mhz is None else int(round(mhz))]
                if isinstance(r2, SnrSweep):
                    snr = r2.compact_summary()
                del r2
                torch.cuda.empty_cache()

    e2e = None
    if not args.no_e2e:
        try:
            e2e = e2e_measure(r, max(2, min(args.steps, 5)))
            e2e["value"] *= world
        except NotImplementedError as exc:   # workloads timed on device tensors only
            e2e = {"unavailable": str(exc)}

    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, on device)",
            "config": dict(describe(args.workload), parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
            "roofline": rf, "e2e": e2e, "gpu_launches": r.launches_per_step * args.steps,
            "clocks": clocks, "sustained": sustained}
    if rank == 0 and not args.no_cpu_baseline and not dist_on:
        line["cpu_baseline"] = cpu_oracle_run(args.workload)
    if snr is not None:
        line["snr_cols"] = ["N", "snr_plain", "snr_diff", "noise_frac_plain"]   # medians over the instances
        line["snr"] = snr
    if secondary:   # last, so that a reader keeping only the end of the line keeps every row
        line["secondary_cols"] = SECONDARY_COLS
        line["secondary"] = secondary
    if rank == 0:
        print(json.dumps(_rounded(line, 5)))
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
