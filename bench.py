#!/usr/bin/env python
"""Benchmark of the W4A4 + low-rank linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl svdq|reference]
                    [--workload mlp_up|qkv|mlp_down|tiny] [--format nvfp4|int4] [--rank R]

One step = the whole hot path on one batch: the prologue (smooth, quantize,
down-project) and the fused W4A4 GEMM (+ up-projection + bias), i.e. one
forward of the DiT MLP-up layer 4608 x 3072 x 12288, rank 32, NVFP4 by
default.  Inputs are seeded synthetic data (bit_w4a4_quantized_group_b200/inputs.py);
weights are
decomposed offline (not timed).  Each timed step is bracketed by CUDA events
on the launching stream; a 512 MB write between steps flushes the 126 MB L2
outside the events.  Multi-GPU runs (torchrun) are independent replicas, one
layer per GPU (weak scaling); time is the max over ranks.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4+low-rank linear effective TFLOPS"
UNIT = "TFLOP/s"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="svdq", choices=["svdq", "reference"])
    ap.add_argument("--workload", default="mlp_up")
    ap.add_argument("--format", default="nvfp4", choices=["nvfp4", "int4", "mxfp4", "w8a8"],
                    help="w8a8 is the 8-bit setting (per-token activations, per-channel weights); "
                         "its rank defaults to 16")
    ap.add_argument("--rank", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--weights", default="svd", choices=["svd", "random"],
                    help="svd: smoothing + SVD split of the synthetic W (default); random: seeded random "
                         "R, L1, L2 of the same shapes and scale, no decomposition (for short profiler runs; "
                         "the kernels' time and traffic do not depend on the weight values)")
    ap.add_argument("--residual-iters", type=int, default=1,
                    help="outer residual iterations of the offline split (1: plain SVD split)")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the headline line, time the layer over the batch x shape x rank grid "
                         "(random weights of each shape) and print one JSON line per point")
    ap.add_argument("--residual-early-stop", action="store_true",
                    help="keep the best residual-iteration candidate and stop once the target gets worse")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), \
            float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 1400.0, FALLBACK_HBM_GBS, "fallback"


def workload(args):
    from bit_w4a4_quantized_group_b200 import inputs as I
    cfg = I.NAMED[args.workload]
    if args.rank is None and args.format == "w8a8":
        args.rank = 16                       # the 8-bit setting's rank
    if args.rank is not None and args.rank != cfg.rank:
        import dataclasses
        cfg = dataclasses.replace(cfg, rank=args.rank)
    return cfg


def prepare_layer(cfg, fmt, device, weights="svd", residual_iters=1, early_stop=False):
    from bit_w4a4_quantized_group_b200 import inputs as I
    from bit_w4a4_quantized_group_b200 import prepare as P
    import torch
    layer = I.make_layer(cfg)
    if weights == "svd":
        if device.startswith("cuda"):
            torch.cuda.synchronize()
        t0 = time.perf_counter()
        prep = P.prepare(fmt, layer.X, layer.W, cfg.rank, device=device,
                         residual_iters=residual_iters, early_stop=early_stop)
        if device.startswith("cuda"):
            torch.cuda.synchronize()
        prep["offline_s"] = time.perf_counter() - t0
    else:
        rng = np.random.default_rng(cfg.seed + 1000)
        K, N, r = cfg.m, cfg.n, cfg.rank
        lam = np.ones(K, np.float32)
        xa = float(np.abs(layer.X).max())
        prep = {"lam": lam,
                "R_nk": (rng.standard_normal((N, K)) * cfg.sigma_w).astype(np.float32),
                "L1_rk": (rng.standard_normal((r, K)) * 0.05).astype(np.float32),
                "L2_nr": (rng.standard_normal((N, r)) * 0.05).astype(np.float32),
                "act_gscale": P.pow2_tensor_scale(xa) if fmt == "nvfp4" else 1.0}   # MXFP4, INT4: none
    packed = P.pack(fmt, prep)
    return layer, prep, packed


class ClockSampler:
    """SM clocks and throttle reasons of one GPU, sampled while the timed steps run.

    Polls NVML from a thread every 5 ms (one sample right at start and one at
    stop, so even a region of a few milliseconds has samples); falls back to
    `nvidia-smi -lms 200` if NVML cannot be used.
    """
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index, uuid=None, pci=None, period_s=0.005):
        self.gpu = gpu_index
        self.uuid = uuid
        self.pci = pci
        self.period = period_s
        self.samples = []          # (sm_mhz, max_mhz, reasons bitmask names)
        self.proc = self.path = self.thread = None
        self._stop = None

    def _nvml_handle(self):
        """The NVML handle of this process's CUDA device (by UUID, then PCI id; CUDA_VISIBLE_DEVICES
        renumbers devices, so the CUDA index is the last resort)."""
        import pynvml as N
        N.nvmlInit()
        if self.uuid:
            try:
                u = self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid
                return N, N.nvmlDeviceGetHandleByUUID(u)
            except Exception:
                pass
        if self.pci:
            try:
                return N, N.nvmlDeviceGetHandleByPciBusId(self.pci)
            except Exception:
                pass
        return N, N.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading
        try:
            N, h = self._nvml_handle()
            bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}
            mx = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))

            def sample():
                sm = float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM))
                r = int(N.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((sm, mx, tuple(n for n, b in bits.items() if r & b)))

            self._stop = threading.Event()
            sample()

            def loop():
                while not self._stop.wait(self.period):
                    sample()
                sample()

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = "nvml"
            return
        except Exception:
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None

    def _read_smi(self):
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        self.samples.append((float(parts[1]), float(parts[2]),
                                             tuple(self.NAMES[i] for i in range(4)
                                                   if parts[5 + i].lower() == "active")))
            os.unlink(self.path)
        except Exception:
            pass

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self._read_smi()
        if not self.samples:
            return None
        mx = max(s[1] for s in self.samples)
        sm = [s[0] for s in self.samples]
        busy = [v for v in sm if v > 0.5 * mx] or sm
        reasons = sorted({n for s in self.samples for n in s[2]})
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(self.samples), "source": self.source}


def source_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_src, workload_name):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload_name]
        if e["source_sha256_16"] != source_hash(kernel_src):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------------------- CPU reference timing

def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([int(i.get("num_threads", 1)) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def time_oracle(cfg, fmt, prep, X, budget_s=12.0):
    """The CPU reference forward (prologue + GEMM, fp64 NumPy) on a bounded sample of rows.

    The row count doubles until one call takes about a quarter of the budget (or covers
    the whole batch); calls of that size then repeat until the budget is spent.
    """
    import oracle as O
    cores = _oracle_cores()
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], prep["act_gscale"])
    rows = 64

    def run(n, lo=0):
        t0 = time.perf_counter()
        O.layer_forward(fmt, X[lo:lo + n], prep["lam"], prep["act_gscale"], packed, None)
        return time.perf_counter() - t0

    dt = run(rows)
    while dt * 4 < budget_s and rows * 2 <= cfg.b:
        rows *= 2
        dt = run(rows)
    total, calls, done = dt, 1, rows
    while total < budget_s:
        lo = (calls * rows) % max(1, cfg.b - rows + 1)
        total += run(rows, lo)
        calls += 1
        done += rows
    tflops = 2.0 * done * cfg.n * cfg.m / total / 1e12
    return {"value": tflops, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{calls} calls x {rows} of {cfg.b} rows of {cfg.name} ({fmt}, r={cfg.rank}); "
                      f"prologue + GEMM in fp64 NumPy, {total:.1f} s"}, packed


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = workload(args)
    from bit_w4a4_quantized_group_b200 import inputs as I
    import oracle as O
    layer = I.make_layer(cfg)
    prep = O.prepare_layer(args.format, layer.X, layer.W, cfg.rank)
    prep = {"lam": prep["lam"], "R_nk": prep["R_nk"], "L1_rk": prep["L1_rk"], "L2_nr": prep["L2_nr"],
            "act_gscale": prep["act_gscale"]}
    packed = O.pack_weight(args.format, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], prep["act_gscale"])
    rows = min(512, cfg.b)
    for _ in range(args.warmup):
        O.layer_forward(args.format, layer.X[:rows], prep["lam"], prep["act_gscale"], packed, None)
    times = []
    for i in range(args.steps):
        lo = (i * rows) % (cfg.b - rows + 1)
        t0 = time.perf_counter()
        O.layer_forward(args.format, layer.X[lo:lo + rows], prep["lam"], prep["act_gscale"], packed, None)
        times.append(time.perf_counter() - t0)
    t = sum(times) / len(times)
    value = 2.0 * rows * cfg.n * cfg.m / t / 1e12
    cores = _oracle_cores()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, args.format, "host memory (CPU reference)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows} rows of {cfg.b} per step ({cfg.name}, {args.format}, r={cfg.rank})"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))
    return 0


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings: one all_reduce when several ranks run."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(world, flops_per_rank, seconds):
    """Throughput of the whole job: every rank processes flops_per_rank in `seconds` (the slowest rank's time)."""
    return world * flops_per_rank / seconds / 1e12


def layer_algorithmic(fmt, M, K, N, r):
    """Algorithmic bytes of the prologue and of the GEMM, and the GEMM's FLOPs (2MNK + 2MNr).

    Prologue: X (2MK), codes and scales, Z (2Mr), L1 (2rK) and lambda (4K).  GEMM: both
    operands' codes and scales, Z, L2 (2Nr), bias (2N) and Y (2MN).  Codes are half a byte
    per element (W8A8: one); scales one byte per 16 (NVFP4) or 32 (MXFP4) elements, two per
    64 (INT4 fp16), four per row (W8A8 fp32).
    """
    if fmt == "w8a8":
        code, sc = 1.0, lambda rows: 4.0 * rows
    else:
        g = {"nvfp4": 16, "mxfp4": 32, "int4": 64}[fmt]
        per = 2.0 if fmt == "int4" else 1.0
        code, sc = 0.5, (lambda rows: rows * K / g * per)
    pro = 2.0 * M * K + code * M * K + sc(M) + 2.0 * M * r + 2.0 * r * K + 4.0 * K
    gemm = code * (M + N) * K + sc(M) + sc(N) + 2.0 * M * r + 2.0 * N * r + 2.0 * N + 2.0 * M * N
    return pro, gemm, 2.0 * M * N * K + 2.0 * M * N * r


def config_dict(cfg, fmt, l2):
    return {"workload": f"{cfg.name} {cfg.b}x{cfg.m}x{cfg.n} r={cfg.rank} {fmt}", "M": cfg.b, "K": cfg.m,
            "N": cfg.n, "rank": cfg.rank, "format": fmt, "bias": cfg.with_bias, "l2": l2}


# ----------------------------------------------------------------------------- GPU path

def run_sweep(args):
    """Layer time over the batch x shape x rank grid, one JSON line per point.

    Each point uses seeded random weights of its shape (kernel time does not depend on the
    values), the fused layer (prologue + GEMM), the same layer at rank 0 and the unfused
    branch (separate passes on cuBLAS bf16) on top of the rank-0 layer.  L2 is flushed
    between timed calls.
    """
    import torch
    from bit_w4a4_quantized_group_b200 import binding as B
    from bit_w4a4_quantized_group_b200 import build as BUILD
    from bit_w4a4_quantized_group_b200 import inputs as I
    from bit_w4a4_quantized_group_b200 import prepare as P
    from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear
    from bit_w4a4_quantized_group_b200.inputs import bf16_bits
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    BUILD.build()
    B.load()
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    fmt = args.format
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    bf16_burst, _, hbm, peak_src = peaks()
    peak = bf16_burst * (4.0 if fmt in ("nvfp4", "mxfp4") else 2.0)

    def timed(fn, n):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        evs = []
        for _ in range(n):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / n * 1e-3

    for cfg in I.sweep_configs():
        layer = I.make_layer(cfg)
        M, K, N, r = cfg.b, cfg.m, cfg.n, cfg.rank
        rng = np.random.default_rng(cfg.seed + 1000)
        xa = float(np.abs(layer.X).max())
        prep = {"lam": np.ones(K, np.float32),
                "R_nk": (rng.standard_normal((N, K)) * cfg.sigma_w).astype(np.float32),
                "L1_rk": (rng.standard_normal((r, K)) * 0.05).astype(np.float32),
                "L2_nr": (rng.standard_normal((N, r)) * 0.05).astype(np.float32),
                "act_gscale": P.pow2_tensor_scale(xa) if fmt == "nvfp4" else 1.0}
        lin = W4A4LowRankLinear(fmt, N, K, P.pack(fmt, prep), prep["lam"], prep["act_gscale"], layer.bias,
                                device=device)
        X = torch.from_numpy(bf16_bits(layer.X).view(np.int16)).to(device).view(torch.bfloat16)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        n = max(5, args.steps)
        t_layer = timed(lambda: lin.forward(X, Y), n)
        t_pro = timed(lambda: lin.prologue_only(X), n)
        t_gemm = timed(lambda: lin.gemm_only(M, Y), n)
        t_r0 = timed(lambda: (lin.prologue_only(X, rank=0), lin.gemm_only(M, Y, rank=0)), n)
        pro_b, gemm_b, gemm_f = layer_algorithmic(fmt, M, K, N, r)
        # the two kernels run one after the other: each is bound by its own roofline
        t_pro_roof = pro_b / (hbm * 1e9)
        t_gemm_hbm = gemm_b / (hbm * 1e9)
        t_gemm_tc = gemm_f / (peak * 1e12)
        t_roof = t_pro_roof + max(t_gemm_hbm, t_gemm_tc)
        out = {"sweep_point": cfg.name, "format": fmt, "M": M, "K": K, "N": N, "rank": r,
               "lora_rank": cfg.lora_rank, "layer_us": t_layer * 1e6, "prologue_us": t_pro * 1e6,
               "gemm_us": t_gemm * 1e6, "tflops": 2.0 * M * N * K / t_layer / 1e12,
               "gemm_frac": (2.0 * M * N * K + 2.0 * M * N * r) / t_gemm / 1e12 / peak,
               "layer_r0_us": t_r0 * 1e6, "fused_overhead_pct": 100.0 * (t_layer / t_r0 - 1.0),
               "roofline": {"gemm_bound": "hbm" if t_gemm_hbm > t_gemm_tc else "tensor",
                            "layer_roof_us": t_roof * 1e6, "frac": t_roof / t_layer,
                            "gemm_roof_us": max(t_gemm_hbm, t_gemm_tc) * 1e6,
                            "gemm_frac": max(t_gemm_hbm, t_gemm_tc) / t_gemm,
                            "prologue_roof_us": t_pro_roof * 1e6, "prologue_frac": t_pro_roof / t_pro,
                            "peaks": f"{peak_src}: HBM {hbm:.0f} GB/s, tensor {peak:.0f} TFLOP/s"}}
        if r > 0:
            up_scale = lin.act_gscale * lin.w_gscale
            lam_d = torch.ones(K, device=device)

            def unfused():
                lin.prologue_only(X, rank=0)
                lin.gemm_only(M, Y, rank=0)
                xh = (X.float() / lam_d).to(torch.bfloat16)
                Y.addmm_(xh @ lin.L1.t(), lin.L2.t(), alpha=up_scale)
            t_unf = timed(unfused, n)
            out["unfused_layer_us"] = t_unf * 1e6
            out["unfused_overhead_pct"] = 100.0 * (t_unf / t_r0 - 1.0)
        st, site = B.svdq_get_last_device_error(None)
        if st != B.SVDQ_OK:
            raise RuntimeError(f"device error {st} at site {site}")
        print(json.dumps(out), flush=True)
        del lin, X, Y
        torch.cuda.empty_cache()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)

    from bit_w4a4_quantized_group_b200 import binding as B
    from bit_w4a4_quantized_group_b200 import build as BUILD
    from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear
    BUILD.build()
    B.load()

    cfg = workload(args)
    fmt = args.format
    layer, prep, packed = prepare_layer(cfg, fmt, str(device), args.weights, args.residual_iters,
                                        args.residual_early_stop)
    M, K, N, r = cfg.b, cfg.m, cfg.n, cfg.rank
    lin = W4A4LowRankLinear(fmt, N, K, packed, prep["lam"], prep["act_gscale"], layer.bias, device=device)
    from bit_w4a4_quantized_group_b200.inputs import bf16_bits
    X = torch.from_numpy(bf16_bits(layer.X).view(np.int16)).to(device).view(torch.bfloat16)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    # warm-up (untimed)
    for _ in range(args.warmup):
        flush.zero_()
        lin.forward(X, Y)
    barrier()
    st, site = B.svdq_get_last_device_error(None)
    if st != B.SVDQ_OK:
        raise RuntimeError(f"device error {st} at site {site}")

    props = torch.cuda.get_device_properties(local)
    pci = None
    if hasattr(props, "pci_bus_id"):
        pci = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    clocks = ClockSampler(local, uuid=str(getattr(props, "uuid", "")) or None, pci=pci)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    launches = 0
    barrier()
    clocks.start()
    torch.cuda.nvtx.range_push("svdq_timed")
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        lin.prologue_only(X)
        launches += B.svdq_last_launch_count()
        ev[i][1].record(stream)
        lin.gemm_only(M, Y)
        launches += B.svdq_last_launch_count()
        ev[i][2].record(stream)
    barrier()
    torch.cuda.nvtx.range_pop()
    clk = clocks.stop()
    t_pro = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps * 1e-3
    t_gemm = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps * 1e-3
    t_step = t_pro + t_gemm
    steps_us = sorted(e[0].elapsed_time(e[2]) * 1e3 for e in ev)

    def pct(q):
        return steps_us[min(len(steps_us) - 1, int(round(q * (len(steps_us) - 1))))]
    step_dist = {"p10": pct(0.1), "p50": pct(0.5), "p90": pct(0.9)}
    # the same step with a warm L2 (no flush in between): reported beside the headline only
    hot = []
    for i in range(max(5, args.steps // 2)):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        lin.forward(X, Y)
        b.record(stream)
        hot.append((a, b))
    torch.cuda.synchronize()
    t_hot = sum(a.elapsed_time(b) for a, b in hot) / len(hot) * 1e-3

    # low-rank overhead: the same GEMM without the branch (not part of the headline)
    gemm0 = []
    for i in range(max(5, args.steps // 2)):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        lin.gemm_only(M, Y, rank=0)
        b.record(stream)
        gemm0.append((a, b))
    torch.cuda.synchronize()
    t_gemm0 = sum(a.elapsed_time(b) for a, b in gemm0) / len(gemm0) * 1e-3
    # Library reference for the plain 4-bit product (no branch, no bias): cuBLASLt's NVFP4
    # GEMM through torch._scaled_mm on the very same code and scale buffers (the 128x4
    # blocked scale layout is the one cuBLASLt takes).  Context only, not part of any value.
    library = None
    if fmt == "nvfp4" and hasattr(torch, "float4_e2m1fn_x2"):
        try:
            ws = lin.workspace(M)
            A4 = ws["a_codes"].view(torch.float4_e2m1fn_x2).view(M, K // 2)
            W4 = lin.w_codes.view(torch.float4_e2m1fn_x2).view(N, K // 2).t()
            sa = ws["a_scales"].view(torch.float8_e4m3fn)
            sb = lin.w_scales.view(torch.float8_e4m3fn)
            lin.prologue_only(X)
            lin.gemm_only(M, Y, rank=0)
            Yl = torch._scaled_mm(A4, W4, sa, sb, out_dtype=torch.bfloat16)
            Yours = Y.float() - (lin.bias.float() if lin.bias is not None else 0.0)
            rel = float((Yl.float() * (lin.act_gscale * lin.w_gscale) - Yours).norm() / Yours.norm())
            lt = []
            for i in range(args.warmup + max(5, args.steps // 2)):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                torch._scaled_mm(A4, W4, sa, sb, out_dtype=torch.bfloat16)
                b.record(stream)
                if i >= args.warmup:
                    lt.append((a, b))
            torch.cuda.synchronize()
            t_lib = sum(a.elapsed_time(b) for a, b in lt) / len(lt) * 1e-3
            library = {"kernel": "cuBLASLt NVFP4 GEMM (torch._scaled_mm), same operands, rank 0, no bias",
                       "us": t_lib * 1e6, "tflops": 2.0 * M * N * K / t_lib / 1e12,
                       "ours_rank0_us": t_gemm0 * 1e6, "rel_fro_vs_ours": rel}
        except Exception as e:                          # a torch build without the FP4 path
            library = {"unavailable": f"{type(e).__name__}: {str(e)[:120]}"}
    # Fusion: the layer without the branch (prologue and GEMM at rank 0), and the same layer
    # with an unfused branch as separate passes (msModelSlim's two-path forward: the residual
    # linear's output plus two chained low-rank linears): X / lambda -> bf16, Z = X_hat L1^T,
    # Y += Z L2^T, the low-rank products on cuBLAS in bf16.  Reported beside the headline,
    # not part of it.
    fusion = None
    if r > 0:
        lam_d = lin.lam if lin.lam is not None else torch.ones(K, device=device)
        L1d, L2sd = lin.L1, lin.L2
        up_scale = lin.act_gscale * lin.w_gscale          # L2 is stored divided by g_x g_w

        def branch():
            xh = (X.float() / lam_d).to(torch.bfloat16)
            z = xh @ L1d.t()
            Y.addmm_(z, L2sd.t(), alpha=up_scale)

        res = {"r0": [], "unfused": []}
        for i in range(args.warmup + max(5, args.steps // 2)):
            for key in ("r0", "unfused"):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                lin.prologue_only(X, rank=0)
                lin.gemm_only(M, Y, rank=0)
                if key == "unfused":
                    branch()
                b.record(stream)
                if i >= args.warmup:
                    res[key].append((a, b))
        torch.cuda.synchronize()
        t_r0 = sum(a.elapsed_time(b) for a, b in res["r0"]) / len(res["r0"]) * 1e-3
        t_unf = sum(a.elapsed_time(b) for a, b in res["unfused"]) / len(res["unfused"]) * 1e-3
        # the unfused layer computes the same Y (up to bf16 rounding of its extra passes)
        Yu = Y.float().clone()
        lin.forward(X, Y)
        rel = float((Yu - Y.float()).norm() / Y.float().norm())
        fusion = {"t_r0": t_r0, "t_unfused": t_unf, "rel": rel}
    lin.forward(X, Y)                        # restore Y with the branch
    st, site = B.svdq_get_last_device_error(None)
    if st != B.SVDQ_OK:
        raise RuntimeError(f"device error {st} at site {site}")

    # end to end through the public layer API with host buffers
    e2e = None
    if not args.no_e2e:
        Xh = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
        Xh.copy_(X.cpu())
        Yh = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
        for _ in range(2):
            X.copy_(Xh, non_blocking=True)
            lin.forward(X, Y)
            Yh.copy_(Y, non_blocking=True)
        barrier()
        ee = []
        for i in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            X.copy_(Xh, non_blocking=True)
            lin.forward(X, Y)
            Yh.copy_(Y, non_blocking=True)
            b.record(stream)
            ee.append((a, b))
        barrier()
        t_serial = sum(a.elapsed_time(b) for a, b in ee) / len(ee) * 1e-3
        # Pipelined: step i's input copy, layer call and result copy on three streams, so that
        # the copies of neighbouring steps overlap the layer and each other (two device
        # buffers each for X and Y).  Every step still copies its X in and its Y out.
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        Xd = [X, torch.empty_like(X)]
        Yd = [Y, torch.empty_like(Y)]
        Yhs = [Yh, torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)]
        h2d = [torch.cuda.Event() for _ in range(args.steps)]
        comp = [torch.cuda.Event() for _ in range(args.steps)]
        d2h = [torch.cuda.Event() for _ in range(args.steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier()
        t0.record(stream)
        s_in.wait_event(t0)
        for i in range(args.steps):
            bi = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp[i - 2])         # layer i-2 has read X[bi]
                Xd[bi].copy_(Xh, non_blocking=True)
                h2d[i].record(s_in)
            stream.wait_event(h2d[i])
            if i >= 2:
                stream.wait_event(d2h[i - 2])            # Y[bi] of step i-2 has been copied out
            lin.forward(Xd[bi], Yd[bi])
            comp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp[i])
                Yhs[bi].copy_(Yd[bi], non_blocking=True)
                d2h[i].record(s_out)
        stream.wait_event(d2h[args.steps - 1])
        t1.record(stream)
        barrier()
        t_e2e = t0.elapsed_time(t1) / args.steps * 1e-3
        e2e = {"t": t_e2e, "t_serial": t_serial, "h2d": M * K * 2, "d2h": M * N * 2}

    # max over ranks
    t_step, t_pro, t_gemm, t_gemm0, t_e2e, t_e2e_serial, t_r0, t_unf = max_over_ranks(
        [t_step, t_pro, t_gemm, t_gemm0, e2e["t"] if e2e else 0.0, e2e["t_serial"] if e2e else 0.0,
         fusion["t_r0"] if fusion else 0.0, fusion["t_unfused"] if fusion else 0.0], device=device)

    flops = 2.0 * M * N * K
    value = whole_job_tflops(world, flops, t_step)
    bf16_burst, bf16_sus, hbm, peak_src = peaks()
    if fmt in ("nvfp4", "mxfp4"):
        peak = bf16_burst * 4.0              # dense FP4 = 4 x dense bf16 (nominal ratio 9 : 2.25)
        peak_note = f"dense FP4 = 4 x {peak_src} bf16 burst"
        src = os.path.join(ROOT, "bit_w4a4_quantized_group_b200", "csrc", "gemm_nvfp4.cu")
    else:
        peak = bf16_burst * 2.0              # dense INT8 = 2 x dense bf16 (nominal ratio 4.5 : 2.25)
        peak_note = f"dense INT8 = 2 x {peak_src} bf16 burst"
        src = os.path.join(ROOT, "bit_w4a4_quantized_group_b200", "csrc",
                           "gemm_w8a8.cu" if fmt == "w8a8" else "gemm_int4.cu")
    alg_flops = flops + 2.0 * M * N * r
    achieved = alg_flops / t_gemm / 1e12
    traffic = recorded_traffic(src, f"{cfg.name}_{fmt}_r{r}")
    if fmt == "w8a8":
        # algorithmic bytes: X once (the kernel's second pass over X is served mostly from
        # L2), one byte per code, one fp32 scale per row
        pro_bytes = 2 * M * K + M * K + 4 * M + 2 * M * r + 2 * r * K + (4 * K)
    else:
        g = {"nvfp4": 16, "mxfp4": 32, "int4": 64}[fmt]
        sf = 2 if fmt == "int4" else 1
        pro_bytes = 2 * M * K + M * K / 2 + M * K / g * sf + 2 * M * r + 2 * r * K + (4 * K)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": fmt,
        "data": "synthetic" if args.weights == "svd" else "synthetic, random weights (no SVD split)",
        "config": config_dict(cfg, fmt, "flushed: 512 MB write between timed steps, outside the events"),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": f"gemm_{fmt}",
                     "peak_source": peak_note},
        "gemm_us": t_gemm * 1e6, "prologue_us": t_pro * 1e6, "gemm_r0_us": t_gemm0 * 1e6,
        "lowrank_overhead_pct": 100.0 * (t_gemm / t_gemm0 - 1.0),
        "gemm_frac_fp4_peak": (flops / t_gemm / 1e12) / peak,
        "prologue": {"bound": "hbm", "GB/s": pro_bytes / t_pro / 1e9, "peak": hbm,
                     "frac": pro_bytes / t_pro / 1e9 / hbm, "bytes": pro_bytes,
                     "traffic": recorded_traffic(os.path.join(ROOT, "bit_w4a4_quantized_group_b200", "csrc",
                                                              "prologue.cu"),
                                                 f"prologue_{cfg.name}_{fmt}_r{r}")},
        "fusion": None if not fusion else {
            "layer_r0_us": t_r0 * 1e6, "fused_layer_us": t_step * 1e6,
            "fused_overhead_pct": 100.0 * (t_step / t_r0 - 1.0),
            "unfused_layer_us": t_unf * 1e6, "unfused_overhead_pct": 100.0 * (t_unf / t_r0 - 1.0),
            "unfused_branch": "torch bf16 passes: X/lambda, Z = X_hat L1^T, Y += Z L2^T (cuBLAS)",
            "unfused_vs_fused_rel_fro": fusion["rel"]},
        "gpu_launches": launches,
        "clocks": clk,
        "library_reference": library,
        "step_us": step_dist,
        "hot_l2_ms_per_step": t_hot * 1e3,
    }
    if "offline_s" in prep:
        res = prep.get("residual") or {}
        out["offline_split"] = {
            "seconds": prep["offline_s"], "where": str(device), "residual_iters": args.residual_iters,
            "early_stop": args.residual_early_stop, "chosen": res.get("chosen", 0),
            "output_errors": res.get("errors"),
            "note": "smoothing + fp64 SVD split (+ residual iterations), untimed setup, not part of value"}
    if e2e:
        out["e2e"] = {"value": whole_job_tflops(world, flops, t_e2e), "unit": UNIT, "h2d_bytes_per_step": e2e["h2d"],
                      "d2h_bytes_per_step": e2e["d2h"],
                      "copies": "pinned host X in and Y out every step, overlapped across steps on two copy streams",
                      "serial_value": whole_job_tflops(world, flops, t_e2e_serial)}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb, _ = time_oracle(cfg, fmt, prep, layer.X)
        out["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
