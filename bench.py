#!/usr/bin/env python
"""Benchmark of the 4-bit MoE expert-layer numerics on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: routing, NVFP4
quantisation of tokens and expert weights, NVFP4 dispatch, the two NVFP4
grouped GEMMs with SwiGLU and combine, then the backward: MXFP8 quantisation of
the gradients, stochastic requantisation of the saved weights and activations,
MXFP8 dgrad and wgrad grouped GEMMs, SwiGLU backward and un-permute.  The
workload is the 384-expert layer (top-8 of 32768 tokens, d_model 4096, d_ff
1024, Zipf(1.2) loads with 8 empty experts, Student-t(3) activations), synthetic
and seeded.  The step's working set (~40 GB) is far larger than L2, so no
flush is needed between steps.

Multi-GPU: one process per GPU; every rank runs its own replica of the step on
its own tokens (no collective on the data path: weak scaling).  Times are the
max over ranks of CUDA-event device time.

`value` is the NVFP4 grouped-GEMM throughput (both forward GEMMs, flops over
true routed rows) in TFLOP/s, measured inside the timed steps.  The line also
carries the per-stage breakdown, the quantiser bandwidth on the 16384x4096
quantiser stream, the roofline of the dominant kernel, clocks, the end-to-end
number through host buffers, and the CPU oracle baseline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "moe_layer"
QUANT_WORKLOAD = "quant_stream"
METRIC = "NVFP4 grouped expert GEMM TFLOPS (% of B200 FP4 peak); quantiser GB/s (% HBM)"
UNIT = "TFLOP/s"
NOMINAL_NVFP4_TFLOPS = 9000.0
NOMINAL_MXFP8_TFLOPS = 4500.0
NOMINAL_HBM_GBS = 8000.0
SM_MAX_MHZ = 1965.0                   # clocks.max.sm of this machine's B200s
# stages that issue more than one kernel (routing: 4; per-expert NVFP4 weights: amax, quantise, finish;
# the row-mode grouped GEMMs: the CTA-pair kernel and the tail kernel for the experts' leftover row tiles)
MULTI_LAUNCH_STAGES = ("route", "quant_w", "gemm1", "gemm2", "dgrad1", "dgrad2")
# mxfp8_requant_transpose_sr (R = 16) per element, from one ncu capture of `bench.py --kernel requant_w`
# (64 experts x 2048 x 4096, output 0.55 GB > L2): warp-instructions executed and DRAM bytes (read + write)
REQUANT_WARP_INST_PER_ELEM = 0.5966
REQUANT_DRAM_BYTES_PER_ELEM = 1.5817
# DRAM bytes (read + write) of one launch of the step's kernels that are not per-element streams, from one
# ncu capture of `bench.py --steps 1 --warmup 1` (dram__bytes_read.sum + dram__bytes_write.sum, one pass, the
# timed step's launch): wgrad1 reads 3.56 GB and writes the 6.40 GB weight gradient
STAGE_DRAM_BYTES = {"wgrad1": 3558820352 + 6397490944}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons during the timed region: read
    through NVML every 20 ms on a host thread (read-only queries), or, where
    NVML is unavailable, from `nvidia-smi -lms 200`."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.rows = []

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:                                              # the CUDA device's own GPU, whatever the visible set
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[self.gpu].isdigit() else self.gpu
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def __enter__(self):
        import threading
        try:
            import pynvml
            h = self._nvml_handle()
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.stop = threading.Event()

            def loop():
                while not self.stop.is_set():
                    try:
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except Exception:
                        r = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    self.rows.append(dict(sm=float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                          smax=float(smax), power=pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                          reasons={n for b, n in self.REASON_BITS.items() if r & b}))
                    self.stop.wait(0.02)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            return
        out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
        for line in (out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                self.rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]),
                                      reasons={n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown",
                                                                  "sw_thermal_slowdown", "sw_power_cap"), f[5:9])
                                               if v.lower().startswith("active")}))
            except ValueError:
                continue

    def summary(self):
        rows = self.rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples"], "samples": 0}
        loaded = [r for r in rows if r["power"] > 300] or rows
        reasons = set()
        for r in loaded:
            reasons |= r["reasons"]
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded),
                "source": "nvml, 20 ms" if self.thread is not None else "nvidia-smi, 200 ms"}


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, values, device):
    """Element-wise max of a list of floats over ranks."""
    if pg is None:
        return list(values)
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(pg, values, device):
    if pg is None:
        return list(values)
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return t.tolist()


# --------------------------------------------------------------------------
# algorithmic work per stage (bytes read+written once, flops over true rows)
# --------------------------------------------------------------------------
def stage_work(c, counts, M_pad):
    T, k, E, D, F = c["T"], c["k"], c["E"], c["D"], c["F"]
    N1 = 2 * F if c["gated"] else F
    R = T * k                                       # true routed rows
    nv = lambda rows, cols: rows * cols * (0.5 + 1 / 16) + rows * 4          # NVFP4 bytes (+ outer)
    mx = lambda rows, cols: rows * cols * (1 + 1 / 32)                       # MXFP8 bytes
    f_g1 = 2 * R * N1 * D
    f_g2 = 2 * R * D * F
    w = {
        # name: (kind, work)  kind: "tensor4" / "tensor8" flops, "hbm" bytes
        "route": ("hbm", T * k * 4 * 2 + (T * k + 127 * E) * 4),
        "quant_x": ("hbm", T * D * 2 + nv(T, D)),
        "gather": ("hbm", 2 * nv(R, D)),
        "quant_w": ("hbm", E * N1 * D * 2 + nv(E * N1, D) + E * D * F * 2 + nv(E * D, F)),
        "gemm1": ("tensor4", f_g1),
        "swiglu": ("hbm", R * N1 * 2 + R * F * 2),
        "quant_a": ("hbm", R * F * 2 + nv(R, F)),
        "swiglu_quant": ("hbm", R * N1 * 2 + nv(R, F)),          # SwiGLU + NVFP4 in one kernel
        "gemm2": ("tensor4", f_g2),
        "combine": ("hbm", R * D * 2 + T * D * 2),
        "dispatch_grad": ("hbm", T * D * 2 + R * D * 2),
        "quant_dy2": ("hbm", R * D * 2 + 2 * mx(R, D)),
        "dispatch_grad_quant": ("hbm", T * D * 2 + 2 * mx(R, D)),  # dispatch gradient + MXFP8 in one kernel
        "requant_w2": ("alu", (nv(E * D, F) + mx(E * D, F), (E * D) * (F))),
        "dgrad2": ("tensor8", 2 * R * F * D),
        "requant_a": ("alu", (nv(R, F) + mx(R, F), (R) * (F))),
        "wgrad2": ("tensor8", 2 * R * D * F),
        "swiglu_bwd": ("hbm", R * N1 * 2 + R * F * 2 + R * N1 * 2),
        "quant_dh1": ("hbm", R * N1 * 2 + 2 * mx(R, N1)),
        "requant_w1": ("alu", (nv(E * N1, D) + mx(E * N1, D), (E * N1) * (D))),
        "dgrad1": ("tensor8", 2 * R * D * N1),
        "requant_x": ("alu", (nv(R, D) + mx(R, D), (R) * (D))),
        "wgrad1": ("tensor8", 2 * R * N1 * D),
        "unpermute": ("hbm", R * D * 2 + T * D * 2),
    }
    return w



def run_ours(args):
    import torch
    from fp8_moe_numerics_b200 import api, workloads
    from fp8_moe_numerics_b200.layer import ExpertLayer

    rank, world, local, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    c = workloads.CONFIGS[WORKLOAD]
    # each rank draws its own tokens (weak scaling); weights are shared seeds
    inp = workloads.layer_inputs(WORKLOAD, device=dev)
    if rank:
        inp["x"] = workloads.activations(c["T"], c["D"], c["x_dist"], c["seed"] + 1 + 1000 * rank, dev)
    topk = inp["topk"].to(dev)
    counts = torch.bincount(inp["topk"].reshape(-1).long(), minlength=c["E"]).tolist()
    M_pad = sum((x + 127) // 128 * 128 for x in counts)
    layer = ExpertLayer(inp["x"], topk, inp["w_comb"].to(dev), inp["w1"], inp["w2"], inp["dout"], gated=c["gated"],
                        seed=1234)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        layer.step()
    api.sync_status()
    torch.cuda.synchronize()

    # ---------------------------------------------------------------- timed
    layer.reset_marks()
    barrier(pg)
    torch.cuda.synchronize()
    from fp8_moe_numerics_b200 import _lib
    launches0 = _lib.lib().mx_kernel_launches()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            layer.step(record=True)
        t1.record(stream)
        torch.cuda.synchronize()
    launches = _lib.lib().mx_kernel_launches() - launches0      # this library's kernels in the timed region
    barrier(pg)
    api.sync_status()
    total_ms = t0.elapsed_time(t1)
    stages = layer.stage_times_ms()
    work = stage_work(c, counts, M_pad)
    names = [n for n in work if n in stages]            # the stages this layer configuration ran
    stage_ms = [stages.get(n, 0.0) for n in names]
    maxed = max_over_ranks(pg, [total_ms] + stage_ms, dev)
    total_ms, stage_ms = maxed[0], dict(zip(names, maxed[1:]))
    K = args.steps
    gemm_flops = (work["gemm1"][1] + work["gemm2"][1]) * K
    nvfp4_ms = stage_ms["gemm1"] + stage_ms["gemm2"]
    value = world * gemm_flops / (nvfp4_ms * 1e-3) / 1e12

    # roofline of the dominant kernel: the longest stage that is one launch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    issue_peak = sms * 4 * SM_MAX_MHZ * 1e6 / 1e9           # warp-instructions per ns = G/s
    dom = max((n for n in names if n not in MULTI_LAUNCH_STAGES), key=lambda n: stage_ms[n])
    kind, wk = work[dom]
    per_launch_ms = stage_ms[dom] / K
    if kind == "alu":
        # the requantisation: algorithmic bytes against HBM (the roofline), with the kernel's issue rate
        # (warp-instructions per element from one ncu capture) beside it as a diagnostic
        nbytes, elems = wk
        achieved = nbytes / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4),
                "traffic": round(REQUANT_DRAM_BYTES_PER_ELEM * elems) if REQUANT_DRAM_BYTES_PER_ELEM else None,
                "kernel": dom, "algorithmic_bytes": int(nbytes),
                "peak_source": peaks["src"] + " copy bandwidth",
                "issue_frac": round(REQUANT_WARP_INST_PER_ELEM * elems / (per_launch_ms * 1e-3) / 1e9 / issue_peak, 4),
                "issue_note": f"warp-instructions per element {REQUANT_WARP_INST_PER_ELEM} (ncu) x elements / time, "
                              f"against {sms} SMs x 4 schedulers x {SM_MAX_MHZ} MHz"}
    elif kind == "hbm":
        achieved = wk / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "traffic": None, "kernel": dom, "algorithmic_bytes": int(wk),
                "peak_source": peaks["src"] + " copy bandwidth"}
    else:
        ratio = 4 if kind == "tensor4" else 2
        peak = peaks["bf16_sus"] * ratio
        achieved = wk / (per_launch_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": STAGE_DRAM_BYTES.get(dom), "kernel": dom,
                "algorithmic_flops": int(wk),
                "peak_source": f"{peaks['src']} sustained bf16 x {ratio} (nominal dense ratio)"}
    breakdown = {}
    for n in names:
        kind, wk = work[n]
        t = stage_ms[n] / K
        if kind == "alu":
            nbytes, elems = wk
            breakdown[n] = {"ms": round(t, 4), "GB/s": round(nbytes / (t * 1e-3) / 1e9, 1) if t > 0 else None,
                            "frac_hbm": round(nbytes / (t * 1e-3) / 1e9 / peaks["hbm"], 3) if t > 0 else None,
                            "frac_issue": round(REQUANT_WARP_INST_PER_ELEM * elems / (t * 1e-3) / 1e9 / issue_peak, 3)
                            if t > 0 else None}
        elif kind == "hbm":
            breakdown[n] = {"ms": round(t, 4), "GB/s": round(wk / (t * 1e-3) / 1e9, 1) if t > 0 else None,
                            "frac_hbm": round(wk / (t * 1e-3) / 1e9 / peaks["hbm"], 3) if t > 0 else None}
        else:
            ratio = 4 if kind == "tensor4" else 2
            tf = wk / (t * 1e-3) / 1e12 if t > 0 else None
            breakdown[n] = {"ms": round(t, 4), "TFLOP/s": round(tf, 1) if tf else None,
                            "frac_nominal": round(tf / (NOMINAL_NVFP4_TFLOPS if ratio == 4 else NOMINAL_MXFP8_TFLOPS), 3)
                            if tf else None,
                            "frac_measured": round(tf / (peaks["bf16_sus"] * ratio), 3) if tf else None}

    quant = quantiser_stream(dev, peaks) if rank == 0 else None
    s2f6 = combine_s2f6_leg(layer, c, counts, peaks) if rank == 0 else None
    mx_fwd = mxfp8_forward_leg(layer, counts, peaks, breakdown) if rank == 0 else None

    # ---------------------------------------------------------------- e2e
    e2e = e2e_leg(layer, inp, dev, args, gemm_flops / K, pg, world)
    cpu_sample = {"x": inp["x"][:256].cpu(), "w1": inp["w1"][0:1, :256].cpu()}

    # the 64-expert layer's forward GEMMs and backward, after the 384-expert layer's buffers are released
    del layer, inp, topk
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    cfg_legs = gemm_config_legs(dev, peaks) if rank == 0 else None
    torch.cuda.empty_cache()
    nv_bwd = nvfp4_backward_leg(dev, peaks) if rank == 0 else None

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4/mxfp8 (fp32 accumulate), bf16 i/o", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: 384 experts, top-8 of 32768 tokens (262144 routed rows, "
                               f"{M_pad} padded), d_model 4096, d_ff 1024 SwiGLU, Zipf(1.2) loads with 8 empty "
                               "experts, t(3) activations; NVFP4 forward + MXFP8-SR backward",
                   "parallelism": f"replicas x{world} (one per GPU, no data-path collective)",
                   "l2": "per-step working set ~40 GB >> 126 MB L2 (no flush needed)",
                   "seed": c["seed"], "sr_rbits": 16},
        "nvfp4_gemm": {"tflops": round(value / world, 1), "frac_of_9pf_nominal": round(value / world / NOMINAL_NVFP4_TFLOPS, 4),
                       "frac_of_measured": round(value / world / (peaks["bf16_sus"] * 4), 4),
                       "peak_measured_basis": f"{peaks['src']} bf16 sustained {peaks['bf16_sus']} x4"},
        "stages": breakdown,
        "quantiser": quant,
        "combine_s2f6": s2f6,
        "mxfp8_forward": mx_fwd,
        "fwd_gemm": cfg_legs["fwd_gemm"] if cfg_legs else None,
        "bwd_gemm": cfg_legs["bwd_gemm"] if cfg_legs else None,
        "nvfp4_backward": nv_bwd,
        "roofline": roof,
        "clocks": clk.summary(),
        "e2e": e2e,
        "gpu_launches": int(launches),
        "impl": "ours",
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cpu_sample, seconds=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def quantiser_stream(dev, peaks, reps: int = 20):
    """NVFP4 quantise, Hadamard + S2F6 quantise and MXFP8 stochastic
    requantise-transpose of the 16384x4096 Student-t(4) stream; L2 flushed
    before every launch."""
    import torch
    from fp8_moe_numerics_b200 import api, workloads
    c = workloads.CONFIGS[QUANT_WORKLOAD]
    rows, cols = c["rows"], c["cols"]
    x = workloads.activations(rows, cols, c["x_dist"], c["seed"], dev)
    q = api.nvfp4_quantize(x, 1, api.MX_SF_MMA)
    t = api.mxfp8_requant_transpose_sr(*q, rows, cols, 1, api.MX_SF_MMA, None, c["sr_seed"], 0, 16, api.MX_SF_MMA)
    # L2 is flushed by READING a 512 MB buffer (a reduction): zeroing it instead would leave up to
    # 126 MB of dirty lines that the next, timed launch writes back
    flush = torch.ones(64 << 20, dtype=torch.int64, device=dev)
    hs = api.hadamard_s2f6_quantize(x, c["sr_seed"], 101)
    res = {}
    for name, fn, nbytes in (
            ("nvfp4_quantize", lambda: api.nvfp4_quantize(x, 1, api.MX_SF_MMA, out=q),
             rows * cols * 2 + rows * cols * (0.5 + 1 / 16) + rows * 4),
            ("hadamard_s2f6_quantize", lambda: api.hadamard_s2f6_quantize(x, c["sr_seed"], 101, out=hs),
             rows * cols * 2 + rows * cols * (1 + 1 / 32)),
            ("mxfp8_requant_transpose_sr", lambda: api.mxfp8_requant_transpose_sr(
                *q, rows, cols, 1, api.MX_SF_MMA, None, c["sr_seed"], 0, 16, api.MX_SF_MMA, out=t),
             rows * cols * (0.5 + 1 / 16) + rows * 4 + rows * cols * (1 + 1 / 32))):
        for _ in range(3):
            fn()
        ms = []
        for _ in range(reps):
            flush.sum()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        med = statistics.median(ms)
        gbs = nbytes / (med * 1e-3) / 1e9
        res[name] = {"us": round(med * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm_measured": round(gbs / peaks["hbm"], 3),
                     "frac_hbm_8tbs": round(gbs / NOMINAL_HBM_GBS, 3), "bytes": int(nbytes)}
    res["workload"] = ("quant_stream: bf16 16384x4096 Student-t(4) x 10^U(-3,3) per row; L2 flushed before every "
                       "launch by a read-only pass over 512 MB; median of 20")
    return res


def combine_s2f6_leg(layer, c, counts, peaks, reps: int = 10):
    """The combine path in S2F6 beside the bf16 one, on the layer's own
    operands after the timed steps: GEMM2 with the bf16 epilogue vs the
    rotate + S2F6 epilogue, and the combine reading bf16 vs S2F6 rows."""
    import torch
    from fp8_moe_numerics_b200 import api
    L = layer
    E, D, F, T, k, M = L.E, L.D, L.F, L.T, L.k, L.M_cap
    seed, sid = c["seed"], 101
    codes = torch.empty(M, D, dtype=torch.int8, device=L.dev)
    e8 = torch.empty(M, D // 32, dtype=torch.uint8, device=L.dev)
    rows = int(sum(int(x) for x in counts))
    flops = 2 * rows * D * F
    legs = (
        ("gemm2_bf16", lambda: api.grouped_gemm_nvfp4(L.aq, L.w2q, L.seg, E, D, F, out=L.y2), "flops", flops),
        ("gemm2_s2f6", lambda: api.grouped_gemm_nvfp4_s2f6(L.aq, L.w2q, L.seg, E, D, F, seed, sid, out=(codes, e8)),
         "flops", flops),
        ("combine_bf16", lambda: api.moe_combine(L.y2, L.pos, L.w_comb, D, out=L.out), "bytes",
         T * k * D * 2 + T * D * 2 + T * k * 8),
        ("combine_s2f6", lambda: api.moe_combine_s2f6(codes, e8, L.pos, L.w_comb, seed, sid, out=L.out), "bytes",
         T * k * (D + D // 32) + T * D * 2 + T * k * 8),
    )
    res = {}
    for name, fn, kind, work in legs:
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        if kind == "flops":
            res[name] = {"ms": round(ms, 4), "TFLOP/s": round(work / (ms * 1e-3) / 1e12, 1)}
        else:
            gbs = work / (ms * 1e-3) / 1e9
            res[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm"], 3)}
    api.sync_status()
    res["bytes_y2"] = {"bf16": M * D * 2, "s2f6": M * D + M * D // 32}
    res["note"] = ("32-d random Hadamard + block-scaled S2F6 in GEMM2's epilogue and the combine reading it, "
                   f"on the layer's operands ({reps} back-to-back launches each)")
    return res


def mxfp8_forward_leg(layer, counts, peaks, breakdown, reps: int = 10):
    """The pages' comparison on this GPU: the two forward expert GEMMs with
    MXFP8 operands (E8M0 per 32, RNE) instead of NVFP4, on the layer's own
    activations and weights, through the MXFP8 row GEMM (weights laid out
    [N, E*K]); against the NVFP4 GEMM times of the timed steps."""
    import torch
    from fp8_moe_numerics_b200 import api
    L = layer
    E, D, F, N1, k, M = L.E, L.D, L.F, L.N1, L.k, L.M_cap
    rows = int(sum(int(x) for x in counts))
    idx = (L.src.clamp(min=0) // k).long()
    res = {}
    a_act = api.swiglu_fwd(L.h1, F, L.gated, L.rows_valid)              # the bf16 activation GEMM2 reads
    for name, a_bf16, w, N, K in (("gemm1", None, L.w1, N1, D), ("gemm2", a_act, L.w2, D, F)):
        if a_bf16 is None:
            a_bf16 = L.x[idx]
            a_bf16[L.src < 0] = 0
        aq = api.mxfp8_quantize(a_bf16, col=False)
        wq = api.mxfp8_quantize(w.permute(1, 0, 2).reshape(N, E * K).contiguous(), col=False)
        out = torch.empty(M, N, dtype=torch.bfloat16, device=L.dev)
        fn = lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, aq[0], aq[1], wq[0], wq[1], L.seg, E, M, N, K, out=out)
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        tf = 2 * rows * N * K / (ms * 1e-3) / 1e12
        nv = breakdown[name]
        res[name] = {"mxfp8_ms": round(ms, 4), "mxfp8_TFLOP/s": round(tf, 1), "nvfp4_ms": nv["ms"],
                     "nvfp4_TFLOP/s": nv["TFLOP/s"], "nvfp4_speedup": round(ms / nv["ms"], 3)}
        del aq, wq, out
    api.sync_status()
    res["note"] = ("forward expert GEMMs with MXFP8 operands on the same layer, 10 back-to-back launches each, "
                   "vs the NVFP4 GEMMs of the timed steps (quantisation not included on either side)")
    return res


def gemm_config_legs(dev, peaks, steps: int = 3, warmup: int = 2):
    """The 64-expert layer (top-8 of 16384 tokens, Zipf(1.1), d_model 4096,
    d_ff 1536 SwiGLU, N(0,1) tokens): its two NVFP4 forward GEMMs, and its
    backward (requantisation of the saved NVFP4 operands, MXFP8 dgrad and wgrad)
    on an upstream gradient N(0, 1e-3).  Whole layer steps, each stage timed by
    CUDA events as in the main step."""
    import torch
    from fp8_moe_numerics_b200 import api, workloads
    from fp8_moe_numerics_b200.layer import ExpertLayer
    c, cb = workloads.CONFIGS["fwd_gemm"], workloads.CONFIGS["bwd_gemm"]
    inp = workloads.layer_inputs("fwd_gemm", device=dev)
    T, k, E, D, F = c["T"], c["k"], c["E"], c["D"], c["F"]
    dout = workloads.gradient(T, D, cb["grad_std"], cb["seed"] + 4, dev)
    layer = ExpertLayer(inp["x"], inp["topk"].to(dev), inp["w_comb"].to(dev), inp["w1"], inp["w2"], dout,
                        gated=c["gated"], seed=c["seed"])
    counts = torch.bincount(inp["topk"].reshape(-1).long(), minlength=E).tolist()
    M_pad = sum((x + 127) // 128 * 128 for x in counts)
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    layer.reset_marks()
    for _ in range(steps):
        layer.step(record=True)
    torch.cuda.synchronize()
    api.sync_status()
    st = layer.stage_times_ms()
    work = stage_work(c, counts, M_pad)
    out = {}
    for n, (kind, wk) in work.items():
        if n not in st:
            continue
        t = st[n] / steps
        if kind in ("tensor4", "tensor8"):
            ratio = 4 if kind == "tensor4" else 2
            tf = wk / (t * 1e-3) / 1e12
            out[n] = {"ms": round(t, 4), "TFLOP/s": round(tf, 1),
                      "frac_nominal": round(tf / (NOMINAL_NVFP4_TFLOPS if ratio == 4 else NOMINAL_MXFP8_TFLOPS), 4),
                      "frac_measured": round(tf / (peaks["bf16_sus"] * ratio), 4)}
        else:
            nbytes = wk[0] if kind == "alu" else wk
            gbs = nbytes / (t * 1e-3) / 1e9
            out[n] = {"ms": round(t, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm"], 4)}

    def total(names, kind):
        ms = sum(out[n]["ms"] for n in names)
        if kind == "flops":
            tf = sum(work[n][1] for n in names) / (ms * 1e-3) / 1e12
            return {"ms": round(ms, 4), "TFLOP/s": round(tf, 1)}
        gbs = sum(work[n][1][0] for n in names) / (ms * 1e-3) / 1e9
        return {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm"], 4)}

    fwd = total(("gemm1", "gemm2"), "flops")
    fwd["frac_of_9pf_nominal"] = round(fwd["TFLOP/s"] / NOMINAL_NVFP4_TFLOPS, 4)
    fwd["frac_measured"] = round(fwd["TFLOP/s"] / (peaks["bf16_sus"] * 4), 4)
    bwd = total(("dgrad2", "wgrad2", "dgrad1", "wgrad1"), "flops")
    bwd["frac_of_4p5pf_nominal"] = round(bwd["TFLOP/s"] / NOMINAL_MXFP8_TFLOPS, 4)
    bwd["frac_measured"] = round(bwd["TFLOP/s"] / (peaks["bf16_sus"] * 2), 4)
    req = total(("requant_w2", "requant_a", "requant_w1", "requant_x"), "bytes")
    res = {
        "fwd_gemm": {"workload": f"64 experts, top-8 of {T} tokens ({T * k} routed rows, {M_pad} padded), Zipf(1.1), "
                                 "d_model 4096, W1 4096->3072 (SwiGLU), W2 1536->4096, N(0,1) tokens",
                     "nvfp4_gemms": fwd, "gemm1": out["gemm1"], "gemm2": out["gemm2"]},
        "bwd_gemm": {"workload": "the same layer's backward on an upstream gradient N(0,1e-3): requantisation of "
                                 "the saved NVFP4 W1, W2, tokens and activations to MXFP8 with stochastic rounding "
                                 "(R = 16), MXFP8 dgrad and wgrad of both GEMMs (dH1 is the SwiGLU backward of "
                                 "dgrad2's output)",
                     "mxfp8_gemms": bwd, "requant": req,
                     **{n: out[n] for n in ("requant_w2", "dgrad2", "requant_a", "wgrad2", "requant_w1", "dgrad1",
                                            "requant_x", "wgrad1")}},
        "steps": steps,
    }
    del layer, inp, dout
    return res


def nvfp4_backward_leg(dev, peaks, steps: int = 2, warmup: int = 1):
    """The 384-expert layer with the four backward GEMMs in NVFP4 (stochastically
    rounded E2M1 operands, the pages' stated future work) beside the MXFP8
    backward of the timed steps: step time and per-stage times."""
    import torch
    from fp8_moe_numerics_b200 import api, workloads
    from fp8_moe_numerics_b200.layer import ExpertLayer
    c = workloads.CONFIGS[WORKLOAD]
    inp = workloads.layer_inputs(WORKLOAD, device=dev)
    layer = ExpertLayer(inp["x"], inp["topk"].to(dev), inp["w_comb"].to(dev), inp["w1"], inp["w2"], inp["dout"],
                        gated=c["gated"], seed=c["seed"], backward="nvfp4")
    counts = torch.bincount(inp["topk"].reshape(-1).long(), minlength=c["E"]).tolist()
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    layer.reset_marks()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        layer.step(record=True)
    b.record()
    torch.cuda.synchronize()
    api.sync_status()
    st = layer.stage_times_ms()
    T, k, D, F, E = c["T"], c["k"], c["D"], c["F"], c["E"]
    R, N1 = T * k, 2 * F
    M = layer.M_cap
    nv = lambda rows, cols: rows * cols * (0.5 + 1 / 16) + rows * 4
    work = {   # algorithmic bytes (requantisations, quantisers) or flops over true rows (GEMMs)
        "quant_dy2": ("hbm", R * D * 2 + nv(R, D)),
        "requant_w2": ("hbm", 2 * nv(E * D, F)),
        "dgrad2": ("tensor4", 2 * R * F * D),
        "requant_a": ("hbm", R * D * 2 + nv(D, R) + 2 * nv(R, F)),
        "wgrad2": ("tensor4", 2 * R * D * F),
        "quant_dh1": ("hbm", R * N1 * 2 + nv(R, N1)),
        "requant_w1": ("hbm", 2 * nv(E * N1, D)),
        "dgrad1": ("tensor4", 2 * R * D * N1),
        "requant_x": ("hbm", R * N1 * 2 + nv(N1, R) + 2 * nv(R, D)),
        "wgrad1": ("tensor4", 2 * R * N1 * D),
    }
    res = {"ms_per_step": round(a.elapsed_time(b) / steps, 3), "steps": steps,
           "padded_rows": M, "note": "segments padded to 256 rows for the NVFP4 wgrad's K-stage; requant_a and "
           "requant_x are the two transposed wgrad operands of that GEMM (dY^T from bf16, the saved NVFP4 "
           "activations^T); bytes of each stage read once and written once"}
    for n, (kind, wk) in work.items():
        if n not in st:
            continue
        t = st[n] / steps
        if kind == "hbm":
            gbs = wk / (t * 1e-3) / 1e9
            res[n] = {"ms": round(t, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm"], 4)}
        else:
            tf = wk / (t * 1e-3) / 1e12
            res[n] = {"ms": round(t, 4), "TFLOP/s": round(tf, 1), "frac_nominal": round(tf / NOMINAL_NVFP4_TFLOPS, 4),
                      "frac_measured": round(tf / (peaks["bf16_sus"] * 4), 4)}
    del layer, inp
    return res


def e2e_leg(layer, inp, dev, args, flops_per_step, pg, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs (tokens, routing, combine weights, upstream gradient) from
    pinned host memory and reads the layer output and input gradient back
    (layer.host_stream_steps: the copies of neighbouring steps overlap each
    step's kernels)."""
    import torch
    from fp8_moe_numerics_b200.layer import host_stream_steps
    host_in = {n: inp[n].cpu().pin_memory() for n in ("x", "topk", "w_comb", "dout")}
    host_out = {n: torch.empty(getattr(layer, n).shape, dtype=getattr(layer, n).dtype).pin_memory()
                for n in ("out", "dx")}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())

    host_stream_steps(layer, host_in, host_out, 2)
    torch.cuda.synchronize()
    barrier(pg)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    n = max(1, args.steps)
    a.record()
    host_stream_steps(layer, host_in, host_out, n)
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(pg, [a.elapsed_time(b) / n], dev)[0]
    return {"value": round(world * flops_per_step / (ms * 1e-3) / 1e12, 1), "unit": UNIT,
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": n, "note": "NVFP4 GEMM flops per step / whole step time including pinned-host copies "
                                "(copies of neighbouring steps overlap each step's kernels)"}


def cpu_baseline(inp, seconds: float = 15.0):
    """The oracle, as it stands, on the host cores: NVFP4-quantise a sample of
    token rows and expert-weight rows and run the fp64 grouped GEMM of those
    rows against one expert's W1 tile, until ~`seconds` of CPU work."""
    import numpy as np
    import oracle
    import torch
    x = inp["x"][:256].cpu().view(torch.int16).numpy().view(np.uint16)
    w = inp["w1"][0, :256].cpu().view(torch.int16).numpy().view(np.uint16)
    D = x.shape[1]
    N = w.shape[0]
    flops = 0
    t0 = time.perf_counter()
    it = 0
    while time.perf_counter() - t0 < seconds or it == 0:
        a = oracle.nvfp4_quantize(x)
        b = oracle.nvfp4_quantize(w, group_rows=N)
        seg = np.array([0, x.shape[0]], np.int64)
        oracle.grouped_gemm_nvfp4(*a, *b, seg, N)
        flops += 2 * x.shape[0] * N * D
        it += 1
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{it} x (NVFP4 quantise 256x{D} tokens + 256x{D} rows of W1[0], fp64 GEMM 256x{N}x{D})",
            "seconds": round(dt, 2)}


# --------------------------------------------------------------------------
# single-kernel cases for ncu captures (small enough to profile, outputs
# larger than L2 where DRAM traffic is read off)
# --------------------------------------------------------------------------
KERNEL_CASES = ("gemm_nvfp4", "gemm_nvfp4_s2f6", "gemm_nvfp4_down", "gemm_mxfp8_dgrad", "gemm_mxfp8_wgrad", "requant", "requant_w",
                "nvfp4_quantize", "quant_w", "mxfp8_quantize", "nvfp4_quantize_sr", "requant_nvfp4", "requant_nvfp4_w",
                "dispatch_grad_quant", "gemm_nvfp4_wgrad",
                "step_nvfp4_backward", "gemm1_moe_layer", "gemm2_moe_layer")


def run_kernel(args):
    import torch
    from fp8_moe_numerics_b200 import api, workloads
    dev = torch.device("cuda")
    which = args.kernel
    if which == "step_nvfp4_backward":
        # one forward + backward step of the benchmark layer with the four backward GEMMs in NVFP4
        from fp8_moe_numerics_b200.layer import ExpertLayer
        c = workloads.CONFIGS[WORKLOAD]
        inp = workloads.layer_inputs(WORKLOAD, device=dev)
        layer = ExpertLayer(inp["x"], inp["topk"].to(dev), inp["w_comb"].to(dev), inp["w1"], inp["w2"], inp["dout"],
                            gated=c["gated"], seed=c["seed"], backward="nvfp4")
        run = layer.step
    elif which in ("gemm1_moe_layer", "gemm2_moe_layer"):
        # the 384-expert layer's forward GEMMs at their own shapes and routing (262144 routed rows, Zipf 1.2 with
        # 8 empty experts): seeded valid codes and scales (the kernel's time does not depend on their values);
        # about 4 GB on the device
        c = workloads.CONFIGS[WORKLOAD]
        E, T, k, D, F = c["E"], c["T"], c["k"], c["D"], c["F"]
        ids = workloads.routing(T, k, E, c["routing"], c["zipf"], c["n_empty"], c["seed"]).to(dev)
        seg, src, pos = api.moe_route(ids, E)
        M = src.shape[0]
        N, K = (2 * F, D) if which == "gemm1_moe_layer" else (D, F)
        g = torch.Generator(device=dev)
        g.manual_seed(9)
        a = (torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g),
             torch.randint(0x30, 0x48, (M * K // 16,), dtype=torch.uint8, device=dev, generator=g),
             torch.full((M,), 1e-3, device=dev))
        b = (torch.randint(0, 256, (E * N, K // 2), dtype=torch.uint8, device=dev, generator=g),
             torch.randint(0x30, 0x48, (E * N * K // 16,), dtype=torch.uint8, device=dev, generator=g),
             torch.full((E,), 1e-3, device=dev))
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        run = lambda: api.grouped_gemm_nvfp4(a, b, seg, E, N, K, out=out)
    elif which.startswith("gemm"):
        # 64 experts, top-8 of 4096 tokens (Zipf 1.2), d_model 4096, d_ff 1024 (gated)
        E, T, k, D, F = 64, 4096, 8, 4096, 1024
        ids = workloads.routing(T, k, E, "zipf", 1.2, 0, 7).to(dev)
        seg, src, pos = api.moe_route(ids, E)
        M = src.shape[0]
        x = workloads.activations(T, D, "t3", 1, dev)
        xq = api.nvfp4_quantize(x, 1, api.MX_SF_ROWMAJOR)
        xp = api.nvfp4_gather_rows(*xq, src, k, D)
        w1 = workloads.weights(E, 2 * F, D, 0.02, 2, dev).view(E * 2 * F, D)
        w1q = api.nvfp4_quantize(w1, 2 * F, api.MX_SF_MMA)
        if which == "gemm_nvfp4":
            run = lambda: api.grouped_gemm_nvfp4(xp, w1q, seg, E, 2 * F, D)
        elif which in ("gemm_nvfp4_s2f6", "gemm_nvfp4_down"):
            # the down projection (N = d_model, K = d_ff) with the rotate + S2F6 epilogue, or with the bf16
            # epilogue on the same operands
            a = api.nvfp4_quantize(workloads.activations(M, F, "t3", 4, dev), 1, api.MX_SF_MMA)
            w2q = api.nvfp4_quantize(workloads.weights(E, D, F, 0.02, 5, dev).view(E * D, F), D, api.MX_SF_MMA)
            if which == "gemm_nvfp4_s2f6":
                run = lambda: api.grouped_gemm_nvfp4_s2f6(a, w2q, seg, E, D, F, 1, 101)
            else:
                run = lambda: api.grouped_gemm_nvfp4(a, w2q, seg, E, D, F)
        elif which == "gemm_nvfp4_wgrad":
            # dW1 in NVFP4 on the same routing with segments padded to 256 tokens: A = dH^T [2F, M256],
            # B = X^T [D, M256]; valid random codes and scales (the kernel's time does not depend on them)
            cnt = (seg[1:] - seg[:-1]).cpu()
            s256 = torch.zeros(E + 1, dtype=torch.int64)
            s256[1:] = torch.cumsum((cnt + 255) // 256 * 256, 0)
            M2 = int(s256[-1])
            g = torch.Generator(device=dev)
            g.manual_seed(8)
            ops = []
            for rows in (2 * F, D):
                codes = torch.randint(0, 256, (rows, M2 // 2), dtype=torch.uint8, device=dev, generator=g)
                sf = torch.randint(0x30, 0x48, (rows * M2 // 16,), dtype=torch.uint8, device=dev, generator=g)
                ops.append((codes, sf))
            A = (*ops[0], torch.full((E * 2 * F,), 1e-3, device=dev))
            B = (*ops[1], torch.full((E,), 1e-3, device=dev))
            s256 = s256.to(dev)
            run = lambda: api.grouped_gemm_nvfp4_wgrad(A, B, s256, E, 2 * F, D, out_dtype=torch.bfloat16)
        else:
            dh = workloads.gradient(M, 2 * F, 1e-3, 3, dev)
            q = api.mxfp8_quantize(dh)
            if which == "gemm_mxfp8_dgrad":
                w1t = api.mxfp8_requant_transpose_sr(*w1q, E * 2 * F, D, 2 * F, seed=1, stream_id=1)
                run = lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, q[0], q[1], *w1t, seg, E, M, D, 2 * F)
            else:
                xt = api.mxfp8_requant_transpose_sr(*xp, M, D, 1, rows_valid=seg[E:E + 1], seed=1, stream_id=2)
                run = lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, q[2], q[3], *xt, seg, E, M, 2 * F, D)
    elif which in ("requant", "nvfp4_quantize", "nvfp4_quantize_sr", "requant_nvfp4"):
        c = workloads.CONFIGS[QUANT_WORKLOAD]
        x = workloads.activations(c["rows"], c["cols"], c["x_dist"], c["seed"], dev)
        q = api.nvfp4_quantize(x)
        if which == "requant":
            run = lambda: api.mxfp8_requant_transpose_sr(*q, c["rows"], c["cols"], seed=c["sr_seed"])
        elif which == "nvfp4_quantize":
            run = lambda: api.nvfp4_quantize(x, out=q)
        elif which == "nvfp4_quantize_sr":            # NVFP4 backward: E2M1 codes rounded stochastically, R = 16
            run = lambda: api.nvfp4_quantize_sr(x, seed=c["sr_seed"], out=q)
        else:                                           # NVFP4 backward: requantisation across the transpose
            t = api.nvfp4_requant_transpose_sr(*q, c["rows"], c["cols"], seed=c["sr_seed"])
            run = lambda: api.nvfp4_requant_transpose_sr(*q, c["rows"], c["cols"], seed=c["sr_seed"], out=t)
    elif which == "requant_nvfp4_w":
        # NVFP4 backward: 64 experts of 2048 x 4096 weights requantised to the NVFP4 stack of W_e^T,
        # per-expert outer scales
        E, N, K = 64, 2048, 4096
        w = workloads.weights(E, N, K, 0.02, 2, dev).view(E * N, K)
        q = api.nvfp4_quantize(w, N, api.MX_SF_MMA)
        t = api.nvfp4_requant_transpose_sr(*q, E * N, K, N, api.MX_SF_MMA, E, True, seed=1, stream_id=16)
        run = lambda: api.nvfp4_requant_transpose_sr(*q, E * N, K, N, api.MX_SF_MMA, E, True, seed=1, stream_id=16,
                                                     out=t)
    elif which == "dispatch_grad_quant":
        # the dispatch gradient formed inside its MXFP8 quantiser: 64 experts, top-8 of 16384 tokens (Zipf 1.1),
        # d_model 4096 (dout 134 MB, outputs 1.1 GB, both > L2)
        E, T, k, D = 64, 16384, 8, 4096
        ids = workloads.routing(T, k, E, "zipf", 1.1, 0, 7).to(dev)
        seg, src, pos = api.moe_route(ids, E)
        dout = workloads.gradient(T, D, 1.0, 3, dev)
        w = torch.full((T, k), 1.0 / k, device=dev)
        q = api.moe_dispatch_grad_mxfp8_quantize(dout, src, w, k, seg[E:E + 1])
        run = lambda: api.moe_dispatch_grad_mxfp8_quantize(dout, src, w, k, seg[E:E + 1], out=q)
    elif which == "requant_w":
        # 64 experts of 2048 x 4096 weights, per-expert outer scales (output 0.55 GB > L2)
        E, N, K = 64, 2048, 4096
        w = workloads.weights(E, N, K, 0.02, 2, dev).view(E * N, K)
        q = api.nvfp4_quantize(w, N)
        run = lambda: api.mxfp8_requant_transpose_sr(*q, E * N, K, N, seed=1, stream_id=3)
    elif which == "quant_w":
        # per-expert NVFP4 of 64 experts of 2048 x 4096 bf16 weights (1.07 GB > L2)
        E, N, K = 64, 2048, 4096
        w = workloads.weights(E, N, K, 0.02, 2, dev).view(E * N, K)
        q = api.nvfp4_quantize(w, N, api.MX_SF_MMA)
        run = lambda: api.nvfp4_quantize(w, N, api.MX_SF_MMA, out=q)
    else:                                               # mxfp8_quantize, row + column forms, RNE
        x = workloads.gradient(65536, 4096, 1.0, 5, dev)
        run = lambda: api.mxfp8_quantize(x)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    api.sync_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run()
    e1.record()
    torch.cuda.synchronize()
    api.sync_status()
    print(json.dumps({"kernel": which, "ms": round(e0.elapsed_time(e1), 4)}), flush=True)


def run_reference(args):
    """Reference arm: the CPU oracle timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import numpy as np
    import torch
    import oracle
    from fp8_moe_numerics_b200 import workloads
    c = workloads.CONFIGS[WORKLOAD]
    D, F = c["D"], c["F"]
    x = workloads.activations(256, D, c["x_dist"], c["seed"] + 1).view(torch.int16).numpy().view(np.uint16)
    w = workloads.weights(1, 2 * F, D, c["w_std"], c["seed"] + 2)[0, :256].view(torch.int16).numpy().view(np.uint16)
    seg = np.array([0, 256], np.int64)
    per = 2 * 256 * 256 * D

    def step():
        a = oracle.nvfp4_quantize(x)
        b = oracle.nvfp4_quantize(w, group_rows=256)
        oracle.grouped_gemm_nvfp4(*a, *b, seg, 256)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    v = per * args.steps / dt / 1e12
    line = {"metric": METRIC, "value": round(v, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "config": {"workload": f"{WORKLOAD} (bounded sample: 256 token rows x 256 W1 rows, d_model {D})"},
            "impl": "reference",
            "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                             "sample": "per step: NVFP4-quantise 256x4096 tokens and 256x4096 W1 rows, fp64 GEMM"},
            "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=KERNEL_CASES, default=None,
                    help="run one kernel on a small case (warm-up, then one launch) for profiling")
    args = ap.parse_args()
    if args.kernel:
        run_kernel(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
