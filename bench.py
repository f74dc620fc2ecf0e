#!/usr/bin/env python
"""Benchmark of sink-softmax GQA attention on B200.

Workload of one step: the gpt-oss-20b shaped prefill -- B=1, L=4096, Hq=64,
Hkv=8, D=64, bf16 -- as two layers run back to back, one dense causal and one
causal banded to a window of 128 (forward: output bf16 + fp32 LSE).
Metric: prefill TFLOP/s, counting only unmasked scores (4*D flops per visible
(query, key) pair), whole job over all ranks.  Further legs measured in the
same run (rank 0 only), each against its own roof: split-KV decode (B=64
ragged sequences up to 32768, dense and window-128, contiguous and paged) in
KV GB/s; the backward at the prefill shape; forward and backward at the
training shape (B8 L8192); the long-context layers (window 128 at L=131072,
dense at L=32768).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-legs]

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
the same workload (independent problems, no collective on the data path);
`value` is the total work of all ranks over the max-over-ranks device time.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "gpt-oss-20b prefill B1 L4096 Hq64 Hkv8 D64 bf16, dense causal + window-128 layers"
METRIC = "prefill TFLOP/s (unmasked scores, 4*D flop per visible pair), dense+banded layers"
B, L, HQ, HKV, D, WIN = 1, 4096, 64, 8, 64, 128
SCALE = 1.0 / math.sqrt(D)
FLUSH_BYTES = 256 << 20


def n_visible(L_, window):
    """Visible (query, key) pairs of one (b, h) for Lq = Lk = L_."""
    if window <= 0 or window >= L_:
        return L_ * (L_ + 1) // 2
    return window * (window + 1) // 2 + (L_ - window) * window


def fwd_flops(B_, L_, Hq_, window):
    return 4.0 * D * n_visible(L_, window) * B_ * Hq_


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            pk = json.load(fh)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ----------------------------------------------------------------------------- our arm
def make_prefill(seed, dev):
    from gqa_softmax_attention_attn_b200.inputs import prefill_inputs

    t = prefill_inputs(B, L, L, HQ, HKV, D, torch.bfloat16, 0.5, 1.0, 0.1, seed=seed, with_dout=True)
    return {k: v.to(dev) for k, v in t.items()}, t


def kernel_source_sha256(kernel_file: str) -> str:
    """sha256 of a kernel's source file followed by the PTX helper header it includes."""
    csrc = os.path.join(ROOT, "gqa_softmax_attention_attn_b200", "csrc")
    h = hashlib.sha256()
    for f in (kernel_file, "sm100_ptx.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_from_profile(kernel_file: str, profile_json: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it is now (else null)."""
    try:
        with open(os.path.join(ROOT, "profiles", profile_json)) as fh:
            pj = json.load(fh)
        if pj.get("source_sha256") != kernel_source_sha256(kernel_file):
            return None
        return float(pj["dram_bytes_per_launch"])
    except Exception:
        return None


def run_ours(args, rank, world, dev):
    import gqa_softmax_attention_attn_b200 as attn
    from gqa_softmax_attention_attn_b200 import multirank

    hbm, tf_burst, tf_sust, peak_src = peaks()
    stream = torch.cuda.current_stream(dev)
    layers = []
    for li, window in enumerate((0, WIN)):
        d, host = make_prefill(multirank.rank_seed(1002 + li, rank), dev)
        d["out"] = torch.empty_like(d["q"])
        d["lse"] = torch.empty(B, HQ, L, device=dev, dtype=torch.float32)
        d["window"] = window
        d["host"] = host
        layers.append(d)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def launch(d):
        attn.attn_sink_fwd(d["q"], d["k"], d["v"], d["sinks"], d["out"], d["lse"], d["window"], SCALE, stream)

    for _ in range(args.warmup):
        flush.zero_()
        for d in layers:
            launch(d)
    torch.cuda.synchronize(dev)
    assert attn.attn_sink_get_device_status(stream) == 0

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if rank == 0:
        sampler.start()
        time.sleep(0.5)
    multirank.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        launch(layers[0])
        ev[i][1].record(stream)
        launch(layers[1])
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    multirank.barrier()
    if rank == 0:
        time.sleep(0.3)
        sampler.stop()
    dense_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    band_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    step_ms = sum(dense_ms) + sum(band_ms)
    status = attn.attn_sink_get_device_status(stream)
    assert status == 0, f"device status {status}"
    # slowest rank's device times; whole-job rate = all ranks' work over that time
    step_ms, dense_tot, band_tot = multirank.max_over_ranks([step_ms, sum(dense_ms), sum(band_ms)], dev)
    flops_step = fwd_flops(B, L, HQ, 0) + fwd_flops(B, L, HQ, WIN)
    value = multirank.job_throughput(flops_step * K, world, step_ms * 1e-3) / 1e12

    # e2e through the public API with host buffers: attn_sink_fwd_host reads each layer's inputs from
    # pinned host memory and writes its outputs back there, chunk by chunk with the copies overlapped
    e2e = None
    if not args.no_e2e:
        hosts = []
        for d in layers:
            h = {k: d["host"][k].pin_memory() for k in ("q", "k", "v", "sinks")}
            h["out"] = torch.empty(d["out"].shape, dtype=d["out"].dtype).pin_memory()
            h["lse"] = torch.empty(d["lse"].shape, dtype=d["lse"].dtype).pin_memory()
            h["ws"] = torch.empty(attn.attn_sink_fwd_host_workspace_size(B, L, L, HQ, HKV, D), dtype=torch.uint8,
                                  device=dev)
            hosts.append(h)
        h2d = sum(h[k].numel() * h[k].element_size() for h in hosts for k in ("q", "k", "v", "sinks"))
        d2h = sum(h[k].numel() * h[k].element_size() for h in hosts for k in ("out", "lse"))
        Ke = max(3, min(K, 50))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for it in range(Ke + 2):
            if it == 2:
                torch.cuda.synchronize(dev)
                e0.record(stream)
            for d, h in zip(layers, hosts):
                attn.attn_sink_fwd_host(h["q"], h["k"], h["v"], h["sinks"], h["out"], h["lse"], d["window"], SCALE,
                                        h["ws"], E2E_CHUNKS, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = multirank.max_over_ranks([e0.elapsed_time(e1)], dev)[0]
        e2e = {"value": multirank.job_throughput(flops_step * Ke, world, e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "api": "attn_sink_fwd_host",
               "chunks": E2E_CHUNKS}

    dense_avg = dense_tot / K
    achieved = fwd_flops(B, L, HQ, 0) / (dense_avg * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "fwd_tc_kernel (dense causal layer)", "achieved": achieved,
                "peak": tf_burst, "unit": "TFLOP/s", "frac": achieved / tf_burst,
                "peak_source": f"{peak_src} bf16 dense (burst)",
                "traffic": traffic_from_profile("fwd_tc.cu", "fwd_tc_prefill_20b_dense.json")}
    res = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1)*0.5 q/k/v, N(0,1) sinks)",
        "config": {"workload": WORKLOAD, "global_batch": B * world, "seq_len": L, "heads_q": HQ, "heads_kv": HKV,
                   "head_dim": D, "window": WIN, "parallelism": f"dp{world}",
                   "l2": "flushed between steps (256 MB write, outside the timed events)"},
        "roofline": roofline,
        "gpu_launches": 2 * K,
        "e2e": e2e,
        "layers": {"dense_ms": dense_avg, "dense_tflops": achieved,
                   "banded_ms": band_tot / K,
                   "banded_gbs": banded_bytes() / (band_tot / K * 1e-3) / 1e9,
                   "banded_frac_hbm": banded_bytes() / (band_tot / K * 1e-3) / 1e9 / hbm},
    }
    if rank == 0:
        res["clocks"] = sampler.summary(t0, t1)
        res["exp_roof"] = exp_roof(dev, res["clocks"])
    return res


def exp_roof(dev, clocks):
    """The third roof of the dense forward: MUFU ex2 results per second (measured
    by the self-test library's microbenchmark) times the 4*D flop each visible
    pair carries (one exponential per pair; the dense layer evaluates a quarter
    of them on the FMA pipe, which lifts its exp roof by 4/3)."""
    import ctypes

    from gqa_softmax_attention_attn_b200 import build

    try:
        lib = ctypes.CDLL(build.SELFTEST_LIB)
        lib.attn_sink_selftest_pipe_rate.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double)]
        rates = []
        for which in (0, 1):
            r = ctypes.c_double(0.0)
            if lib.attn_sink_selftest_pipe_rate(which, ctypes.byref(r)) != 0:
                return None
            rates.append(r.value)
    except OSError:
        return None
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz") or 0.0
    tf = rates[0] * sms * mhz * 1e6 * 4 * D / 1e12
    return {"ex2_per_clk_per_sm": rates[0], "cvt_bf16x2_per_clk_per_sm": rates[1], "sm_mhz": mhz,
            "exp_roof_tflops": tf, "exp_roof_tflops_dense_cfg": tf * 4 / 3}


def banded_bytes():
    """Compulsory bytes of one banded forward: read q, k, v, sinks; write out (bf16) and lse (fp32)."""
    return (2 * B * L * HQ * D + 2 * 2 * B * L * HKV * D + 4 * HQ + 2 * B * L * HQ * D + 4 * B * HQ * L)


def decode_legs(dev, reps=20, warmup=3, batch=None):
    import gqa_softmax_attention_attn_b200 as attn
    from gqa_softmax_attention_attn_b200.inputs import DECODE, SEEDS, decode_inputs

    hbm, _, _, _ = peaks()
    w = DECODE
    nb = batch or w.B
    d = decode_inputs(nb, w.Lmax, w.Hq, w.Hkv, w.D, w.len_lo, w.len_hi, w.dtype, w.qkv_std, w.sink_std,
                      seed=SEEDS["decode"])
    lens = d["seqlens"].tolist()
    d = {k: v.to(dev) for k, v in d.items()}
    out = torch.empty_like(d["q"])
    lse = torch.empty(nb, w.Hq, device=dev, dtype=torch.float32)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    legs = {}
    for name, window in (("decode_dense", 0), ("decode_window128", WIN)):
        nbytes = attn.attn_sink_decode_workspace_size(nb, w.Hq, w.D, w.Lmax, window, 0)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        kv_rows = sum(min(n, window) if window > 0 else n for n in lens)
        by = kv_rows * w.Hkv * w.D * 2 * 2 + nb * w.Hq * w.D * 2 * 2 + nb * w.Hq * 4 + 4 * nb
        ms = timed(dev, lambda: attn.attn_sink_decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"],
                                                      out, lse, window, SCALE, 0, ws, stream), reps, warmup, flush)
        gbs = by / (ms * 1e-3) / 1e9
        legs[name] = {"ms": ms, "GB/s": gbs, "frac_hbm": gbs / hbm, "bytes": by,
                      "flops": 4.0 * w.D * kv_rows * (w.Hq // w.Hkv) * w.Hkv, "sm_mhz": LEG_CLOCK.last_leg_mhz()}
    # the same caches in FP8 (e4m3 codes, one scale per KV head): half the bytes
    from gqa_softmax_attention_attn_b200.inputs import quantize_e4m3_per_head

    k8, ks = quantize_e4m3_per_head(d["k_cache"])
    v8, vs = quantize_e4m3_per_head(d["v_cache"])
    for name, window in (("decode_fp8_dense", 0), ("decode_fp8_window128", WIN)):
        nbytes = attn.attn_sink_decode_workspace_size(nb, w.Hq, w.D, w.Lmax, window, 0)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        kv_rows = sum(min(n, window) if window > 0 else n for n in lens)
        by = kv_rows * w.Hkv * w.D * 2 + nb * w.Hq * w.D * 2 * 2 + nb * w.Hq * 4 + 4 * nb + 2 * 4 * w.Hkv
        ms = timed(dev, lambda: attn.attn_sink_decode_fp8(d["q"], k8, v8, ks, vs, d["seqlens"], d["sinks"], out, lse,
                                                          window, SCALE, 0, ws, stream), reps, warmup, flush)
        gbs = by / (ms * 1e-3) / 1e9
        legs[name] = {"ms": ms, "GB/s": gbs, "frac_hbm": gbs / hbm, "bytes": by, "kv_dtype": "e4m3",
                      "sm_mhz": LEG_CLOCK.last_leg_mhz()}
    del k8, v8
    # the same caches as a pool of 16-key pages in seeded random order, read
    # through a page table (same compulsory bytes; the table is not credited)
    ps = 16
    maxp = w.Lmax // ps
    n_pages = nb * maxp
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(SEEDS["decode"] + ps)).to(dev)
    kp = torch.empty((n_pages, ps, w.Hkv, w.D), dtype=d["k_cache"].dtype, device=dev)
    vp = torch.empty_like(kp)
    kp[perm] = d["k_cache"].reshape(n_pages, ps, w.Hkv, w.D)
    vp[perm] = d["v_cache"].reshape(n_pages, ps, w.Hkv, w.D)
    table = perm.view(nb, maxp).to(torch.int32).contiguous()
    for name, window in (("decode_paged16_dense", 0), ("decode_paged16_window128", WIN)):
        nbytes = attn.attn_sink_decode_paged_workspace_size(nb, w.Hq, w.D, maxp, ps, window, 0)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        by = legs[name.replace("paged16_", "")]["bytes"]
        ms = timed(dev, lambda: attn.attn_sink_decode_paged(d["q"], kp, vp, table, d["seqlens"], d["sinks"], out,
                                                            lse, window, SCALE, 0, ws, stream), reps, warmup, flush)
        gbs = by / (ms * 1e-3) / 1e9
        legs[name] = {"ms": ms, "GB/s": gbs, "frac_hbm": gbs / hbm, "bytes": by, "page_size": ps,
                      "sm_mhz": LEG_CLOCK.last_leg_mhz()}
    return legs


def fwd_bytes(B_, L_, Hq_, Hkv_):
    """Compulsory bytes of one forward: read q, k, v (bf16), sinks; write out (bf16) and lse (fp32)."""
    return 2 * B_ * L_ * Hq_ * D * 2 + 2 * 2 * B_ * L_ * Hkv_ * D + 4 * Hq_ + 4 * B_ * Hq_ * L_


def bwd_bytes(B_, L_, Hq_, Hkv_):
    """Compulsory bytes of one backward: read q, out, dout (bf16), lse (fp32), k, v, sinks;
    write dq (bf16), dk, dv (bf16), dsinks."""
    return 4 * B_ * L_ * Hq_ * D * 2 + 4 * B_ * L_ * Hkv_ * D * 2 + 4 * B_ * Hq_ * L_ + 8 * Hq_


def device_prefill(B_, L_, Hq_, Hkv_, sink_std, seed, dev, with_dout):
    """Seeded synthetic prefill inputs drawn on the device (q, k, v ~ N(0,1)*0.5 bf16,
    sinks ~ N(0, sink_std^2) fp32, dout ~ N(0,1)*0.1): the bench legs' timing inputs."""
    g = torch.Generator(device=dev).manual_seed(seed)
    t = {"q": (torch.randn(B_, L_, Hq_, D, device=dev, generator=g) * 0.5).to(torch.bfloat16),
         "k": (torch.randn(B_, L_, Hkv_, D, device=dev, generator=g) * 0.5).to(torch.bfloat16),
         "v": (torch.randn(B_, L_, Hkv_, D, device=dev, generator=g) * 0.5).to(torch.bfloat16),
         "sinks": torch.randn(Hq_, device=dev, generator=g) * sink_std}
    if with_dout:
        t["dout"] = (torch.randn(B_, L_, Hq_, D, device=dev, generator=g) * 0.1).to(torch.bfloat16)
    return t


class LegClock:
    """The SM clock read through NVML every ~2 ms while the legs run, so that
    each leg reports the median clock of its own timed repetitions (a leg run
    right after a heavy one can start below the maximum clock)."""

    def __init__(self):
        self.samples, self.window, self.nv = [], None, None
        self.stop_ev = threading.Event()

    def start(self, gpu_index: int):
        try:
            import pynvml

            pynvml.nvmlInit()
            self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.nv = pynvml
        except Exception:
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        while not self.stop_ev.is_set():
            try:
                self.samples.append((time.time(), self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)))
            except Exception:
                pass
            time.sleep(0.002)

    def stop(self):
        if self.nv is not None:
            self.stop_ev.set()
            self.t.join(timeout=2)

    def last_leg_mhz(self):
        if self.window is None:
            return None
        vals = [c for t, c in self.samples if self.window[0] <= t <= self.window[1]]
        return statistics.median(vals) if vals else None


LEG_CLOCK = LegClock()
# chunks of query positions per host-buffer call (transfers overlapped with the kernels); measured on the
# B1 L4096 layers: 1 chunk 1.63 / 1.44 ms (dense / window 128), 2: 1.38 / 1.20, 4: 1.32 / 1.15, 8: 1.46 / 1.26
E2E_CHUNKS = 4
LEG_PAUSE_S = 0.5  # idle time before each leg, so that the previous leg's load does not set its clock


def timed(dev, fn, reps, warmup, flush):
    """Median device time (ms) of fn() over `reps` runs after `warmup`, L2 flushed before each."""
    stream = torch.cuda.current_stream(dev)
    times = []
    torch.cuda.synchronize(dev)
    time.sleep(LEG_PAUSE_S)
    t0 = None
    for it in range(reps + warmup):
        if it == warmup:
            t0 = time.time()
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if it >= warmup:
            times.append(e0.elapsed_time(e1))
    LEG_CLOCK.window = (t0, time.time())
    return statistics.median(times)


def leg_entry(ms, flops, nbytes, bound, shape):
    hbm, tf_burst, _, _ = peaks()
    tf = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    e = {"ms": ms, "TFLOP/s": tf, "frac_tensor": tf / tf_burst, "GB/s": gbs, "frac_hbm": gbs / hbm,
         "flops": flops, "bytes": nbytes, "bound": bound, "shape": shape, "sm_mhz": LEG_CLOCK.last_leg_mhz()}
    e["frac"] = e["frac_hbm"] if bound == "hbm" else e["frac_tensor"]
    return e


def prefill_legs(dev, which=("bwd", "train", "fp8", "varlen", "prologue", "long"), reps=10, warmup=3):
    """Forward / backward legs beyond the headline step, each with its own roofline
    fraction (dense layers against the tensor peak, window-128 layers against HBM),
    L2 flushed before every timed run:
      bwd:   the backward at the prefill shape (B1 L4096 Hq64 Hkv8);
      train: forward and backward at the training shape (B8 L8192 Hq64 Hkv8);
      fp8:   the prefill with e4m3 q, k, v (one scale per head);
      varlen: a prefill batch of 12 packed sequences of mixed lengths;
      prologue: bias + YaRN rotary embedding + split of the prefill's QKV rows;
      long:  the long-context layers (window 128 at L = 131072, dense at L = 32768)."""
    import gqa_softmax_attention_attn_b200 as attn

    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    legs = {}

    def run_shape(prefix, B_, L_, sink_std, seed, windows, do_bwd, do_fwd):
        t = device_prefill(B_, L_, HQ, HKV, sink_std, seed, dev, do_bwd)
        out = torch.empty_like(t["q"])
        lse = torch.empty(B_, HQ, L_, device=dev, dtype=torch.float32)
        shape = f"B{B_} L{L_} Hq{HQ} Hkv{HKV} D{D}"
        if do_bwd:
            dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
            ds = torch.empty(HQ, device=dev, dtype=torch.float32)
            ws = torch.empty(attn.attn_sink_bwd_workspace_size(B_, L_, L_, HQ, HKV, D, attn.DTYPE_BF16),
                             dtype=torch.uint8, device=dev)
        for window in windows:
            tag = "dense" if window <= 0 else "window128"
            bound = "tensor" if window <= 0 else "hbm"
            fwd = lambda: attn.attn_sink_fwd(t["q"], t["k"], t["v"], t["sinks"], out, lse, window, SCALE, stream)
            if do_fwd:
                ms = timed(dev, fwd, reps, warmup, flush)
                legs[f"{prefix}fwd_{tag}"] = leg_entry(ms, fwd_flops(B_, L_, HQ, window), fwd_bytes(B_, L_, HQ, HKV),
                                                       bound, shape)
            if do_bwd:
                fwd()
                bwd = lambda: attn.attn_sink_bwd(t["q"], t["k"], t["v"], t["sinks"], out, t["dout"], lse, dq, dk, dv,
                                                 ds, window, SCALE, ws, stream)
                ms = timed(dev, bwd, reps, warmup, flush)
                legs[f"{prefix}bwd_{tag}"] = leg_entry(ms, 2.5 * fwd_flops(B_, L_, HQ, window),
                                                       bwd_bytes(B_, L_, HQ, HKV), bound, shape)
        assert attn.attn_sink_get_device_status(stream) == 0

    if "bwd" in which:
        run_shape("", B, L, 1.0, 2002, (0, WIN), True, False)
    if "train" in which:
        run_shape("train_", 8, 8192, 1.0, 2003, (0, WIN), True, True)
    if "fp8" in which:
        # the gpt-oss-20b prefill with e4m3 q, k, v (one scale per head), both layers
        from gqa_softmax_attention_attn_b200.inputs import quantize_e4m3_per_head

        t = device_prefill(B, L, HQ, HKV, 1.0, 2009, dev, False)
        q8, qs = quantize_e4m3_per_head(t["q"])
        k8, ks = quantize_e4m3_per_head(t["k"])
        v8, vs = quantize_e4m3_per_head(t["v"])
        out = torch.empty(B, L, HQ, D, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(B, HQ, L, device=dev, dtype=torch.float32)
        shape = f"B{B} L{L} Hq{HQ} Hkv{HKV} D{D}, e4m3 q/k/v"
        nbytes = B * L * HQ * D + 2 * B * L * HKV * D + 4 * (HQ + 2 * HKV) + 2 * B * L * HQ * D + 4 * B * HQ * L
        ws = torch.empty(attn.attn_sink_fwd_fp8_workspace_size(B, L, HKV, D), dtype=torch.uint8, device=dev)
        for window in (0, WIN):
            fn = lambda: attn.attn_sink_fwd_fp8(q8, k8, v8, qs, ks, vs, t["sinks"], out, lse, window, SCALE, ws,
                                                stream)
            ms = timed(dev, fn, reps, warmup, flush)
            tag = "dense" if window <= 0 else "window128"
            e = leg_entry(ms, fwd_flops(B, L, HQ, window), nbytes, "tensor" if window <= 0 else "hbm", shape)
            # the score product runs at the 8-bit rate (twice the bf16 peak), P.V at the 16-bit one
            e["frac_tensor_fp8_qk"] = e["TFLOP/s"] / (2 * peaks()[1])
            legs[f"fp8_fwd_{tag}"] = e
        assert attn.attn_sink_get_device_status(stream) == 0
    if "varlen" in which:
        # a prefill batch of mixed lengths packed back to back (seeded lengths in [256, 4096])
        import numpy as np

        lens = [int(x) for x in np.random.default_rng(1002).integers(256, 4097, 12)]
        tot = sum(lens)
        t = device_prefill(1, tot, HQ, HKV, 1.0, 2007, dev, False)
        q, k, v = t["q"][0], t["k"][0], t["v"][0]
        out = torch.empty_like(q)
        lse = torch.empty(HQ, tot, device=dev, dtype=torch.float32)
        cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=dev)
        shape = f"varlen {len(lens)} seqs, {tot} tokens Hq{HQ} Hkv{HKV} D{D}"
        for window in (0, WIN):
            fn = lambda: attn.attn_sink_fwd_varlen(q, k, v, t["sinks"], out, lse, cu, cu, max(lens), window, SCALE,
                                                   stream)
            ms = timed(dev, fn, reps, warmup, flush)
            fl = sum(fwd_flops(1, n, HQ, window) for n in lens)
            tag = "dense" if window <= 0 else "window128"
            legs[f"varlen_fwd_{tag}"] = leg_entry(ms, fl, fwd_bytes(1, tot, HQ, HKV), "tensor" if window <= 0 else "hbm",
                                                  shape)
        assert attn.attn_sink_get_device_status(stream) == 0
    if "prologue" in which:
        # bias + YaRN rotary embedding + split of the prefill's QKV rows (B1 L4096 Hq64 Hkv8)
        width = (HQ + 2 * HKV) * D
        g = torch.Generator(device=dev).manual_seed(2008)
        qkv = (torch.randn(L, width, device=dev, generator=g) * 0.5).to(torch.bfloat16)
        bias = torch.randn(width, device=dev, generator=g) * 0.1
        pos = torch.arange(L, device=dev, dtype=torch.int32)
        qo = torch.empty(L, HQ, D, dtype=torch.bfloat16, device=dev)
        ko = torch.empty(L, HKV, D, dtype=torch.bfloat16, device=dev)
        vo = torch.empty_like(ko)
        fn = lambda: attn.attn_sink_qkv_prologue(qkv, bias, pos, qo, ko, vo, 150000.0, 32.0, 4096, 32.0, 1.0,
                                                 stream=stream)
        ms = timed(dev, fn, reps, warmup, flush)
        nbytes = 2 * L * width * 2 + 4 * width + 4 * L
        legs["prologue_qkv"] = leg_entry(ms, 0.0, nbytes, "hbm", f"T{L} Hq{HQ} Hkv{HKV} D{D}, YaRN factor 32")
        assert attn.attn_sink_get_device_status(stream) == 0
    if "long" in which:
        run_shape("long_", 1, 131072, 2.0, 2005, (WIN,), False, True)
        run_shape("long_", 1, 32768, 2.0, 2006, (0,), False, True)
    return legs


# ----------------------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(seconds_budget=12.0, seed=1002):
    """Times the fp64 oracle on sampled rows of both layers of the workload.
    Returns (TFLOP/s, threads, description, flops, seconds)."""
    import numpy as np

    import oracle
    from gqa_softmax_attention_attn_b200.inputs import prefill_inputs

    t = prefill_inputs(B, L, L, HQ, HKV, D, torch.bfloat16, 0.5, 1.0, seed=seed)
    rng = np.random.default_rng(seed)
    total_fl, total_s, rows = 0.0, 0.0, 0
    n = 256
    while total_s < seconds_budget:
        for window in (0, WIN):
            ri = rng.integers(0, L, n).astype(np.int32)
            rh = rng.integers(0, HQ, n).astype(np.int32)
            rb = np.zeros(n, dtype=np.int32)
            vis = np.minimum(ri + 1, window) if window > 0 else ri + 1
            t0 = time.perf_counter()
            oracle.fwd_rows(t["q"], t["k"], t["v"], t["sinks"], rb, rh, ri, window, SCALE)
            total_s += time.perf_counter() - t0
            total_fl += 4.0 * D * float(vis.sum())
            rows += n
    desc = (f"{rows} uniformly sampled query rows (dense and window-128 layers) of the {WORKLOAD} workload, "
            f"fp64 oracle, {total_s:.1f} s")
    return total_fl / total_s / 1e12, oracle.num_threads(), desc, total_fl, total_s


_TINY_1CORE = r"""
import json, sys, time
sys.path.insert(0, sys.argv[1])
import torch
import oracle
from gqa_softmax_attention_attn_b200.inputs import prefill_inputs
t = prefill_inputs(1, 256, 256, 8, 2, 64, torch.float32, 1.0, 1.0, seed=1001)
oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, 0.125)  # warm-up (load, first touch)
t0 = time.perf_counter()
for window in (0, 128):
    oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, 0.125)
print(json.dumps({"seconds": time.perf_counter() - t0, "threads": oracle.num_threads()}))
"""


def oracle_tiny_1core():
    """The oracle's forward on the tiny fp32 workload (B1 L256 Hq8 Hkv2 D64, dense and
    window-128 layers) on one host core, in a child process with OMP_NUM_THREADS=1."""
    import subprocess

    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", _TINY_1CORE, ROOT], env=env, capture_output=True, text=True,
                           timeout=300)
        d = json.loads(r.stdout.strip().splitlines()[-1])
    except Exception:
        return None
    flops = fwd_flops(1, 256, 8, 0) + fwd_flops(1, 256, 8, 128)
    return {"workload": "B1 L256 Hq8 Hkv2 D64 fp32, dense + window-128 forward", "seconds": d["seconds"],
            "value": flops / d["seconds"] / 1e12, "unit": "TFLOP/s", "cores": d["threads"]}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    steps = []
    per = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        v, cores, desc, fl, s = oracle_sample(seconds_budget=per, seed=1002 + i)
        if i >= args.warmup:
            steps.append((fl, s))
    fl = sum(x[0] for x in steps)
    s = sum(x[1] for x in steps)
    value = fl / s / 1e12
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s / len(steps) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "global_batch": B, "seq_len": L,
                                             "parallelism": "cpu-oracle"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
                             "tiny_1core": oracle_tiny_1core()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-legs", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["decode", "bwd", "train", "fp8", "varlen", "prologue", "long"], default=None,
                    help="run just one leg (reps = --steps, warm-up = --warmup); used for profiling")
    ap.add_argument("--decode-batch", type=int, default=None, help="sequences in the decode leg (default 64)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from gqa_softmax_attention_attn_b200 import multirank

    rank, world, local = multirank.env_rank()

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        multirank.init("nccl", timeout_s=300)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.only is not None:
        LEG_CLOCK.start(dev.index if dev.index is not None else 0)
        legs = (decode_legs(dev, args.steps, args.warmup, args.decode_batch) if args.only == "decode"
                else prefill_legs(dev, (args.only,), args.steps, args.warmup))
        LEG_CLOCK.stop()
        print(json.dumps({"only": args.only, "legs": legs}), flush=True)
        return
    res = run_ours(args, rank, world, dev)
    if rank == 0:
        if not args.no_legs and world == 1:
            res["legs"] = {}
            LEG_CLOCK.start(dev.index if dev.index is not None else 0)
            res["legs"].update(decode_legs(dev))
            res["legs"].update(prefill_legs(dev))
            LEG_CLOCK.stop()
        if not args.no_cpu_baseline and world == 1:
            v, cores, desc, _, _ = oracle_sample(12.0)
            res["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
                                   "tiny_1core": oracle_tiny_1core()}
        res["device"] = {"name": torch.cuda.get_device_name(dev), "capability": list(torch.cuda.get_device_capability(dev)),
                         "torch": torch.__version__, "cuda": torch.version.cuda}
        print(json.dumps(res), flush=True)
    if world > 1:
        multirank.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
