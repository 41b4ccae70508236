"""Benchmark of the ternary linear hot path of 1.58-bit FLUX on B200.

One step = the whole path on the FLUX.1-dev double-block image-stream QKV
layer (x [4096, 3072] bf16, W [9216, 3072] bf16 -> ternary codes, y [4096,
9216] bf16): absmean quantise/pack of W, then the ternary linear y =
(x . T^T) * s + b.  Inputs are seeded synthetic tensors of that shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  `value` is whole-job throughput in TFLOP/s
(2*M*N*K per step per GPU); multi-GPU runs are independent replicas (each
rank its own tokens and weights; weak scaling, no collective on the data
path).  `--impl reference` times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ternary-linear TFLOP/s & packed-weight GB/s at FLUX shapes; % of roofline"
WORKLOAD = "qkv"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
PROFILE_DIR = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "bit_post_quantised_b200", "csrc")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tern", "reference"], default="tern")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="layer the step runs on (default: the QKV headline; others for profiling)")
    ap.add_argument("--no-extras", action="store_true", help="skip the per-kernel side table")
    ap.add_argument("--fp8", action="store_true",
                    help="run the step on FP8 (E4M3) activations: quantise/pack W, quantise x per token "
                         "row, the kind::f8f6f4 layer (not the headline; no CPU baseline, no side table)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU oracle sample budget (0 skips the CPU baseline, for profiling runs)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {**FALLBACK_PEAKS, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def linear_kernel(layer):
    """(kernel name, source file stem) of the tern_linear launch for this shape
    (the routing of the library's host code)."""
    if layer.M <= 16:
        return "ternary_gemv_kernel", "ternary_gemv"
    if layer.N % 256 == 0:
        return ("ternary_pair_kernel<256>", "ternary_mma2") if layer.M > 64 else \
            ("ternary_tile_kernel<64>", "ternary_mma2")
    return "ternary_mma_kernel", "ternary_mma"


def kernel_source_hash(stem: str) -> str:
    with open(os.path.join(CSRC, stem + ".cu"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(stem: str, workload: str):
    """DRAM bytes per launch of the linear kernel on this workload from the
    committed ncu summary, or None if there is none or the kernel changed since."""
    try:
        text = open(os.path.join(PROFILE_DIR, f"{stem}_{workload}.md")).read()
    except OSError:
        return None
    m_src = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_src or not m_tr or m_src.group(1) != kernel_source_hash(stem):
        return None
    return float(m_tr.group(1))


class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons while the timed
    region runs: NVML every 0.1 ms from a thread (reads only; a timed region
    of a few milliseconds still gets tens of samples), else nvidia-smi every
    100 ms."""

    # NVML clock-event reason bits
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.samples = []  # (sm_mhz, max_mhz, reasons set)
        self.proc = None
        self.thread = None
        self.stop = False
        self.ready = None

    def _nvml_loop(self, handle, nv):
        mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
            except Exception:
                break
            self.samples.append((float(sm), float(mx), {k for k, b in self.REASONS.items() if bits & b}))
            self.ready.set()
            time.sleep(0.0001)

    def __enter__(self):
        try:
            import pynvml as nv

            nv.nvmlInit()
            handle = (nv.nvmlDeviceGetHandleByUUID(self.gpu) if self.gpu.startswith("GPU-")
                      else nv.nvmlDeviceGetHandleByIndex(int(self.gpu)))
            import threading

            self.ready = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(handle, nv), daemon=True)
            self.thread.start()
            # a short timed region must not end before the sampler runs
            self.ready.wait(2.0)
            self.samples.clear()
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
            time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in out.strip().splitlines():
                f = [v.strip() for v in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    self.samples.append((float(f[1]), float(f[2]),
                                         {n for n, v in zip(names, f[5:9]) if v.lower() == "active"}))
                except ValueError:
                    continue

    def summary(self):
        if not self.samples:
            return None
        sm = [a for a, _, _ in self.samples]
        hi = max(sm)
        loaded = [v for v in sm if v >= 0.5 * hi] or sm
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(b for _, b, _ in self.samples),
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvml 0.1 ms" if self.thread is not None else "nvidia-smi 100 ms"}


# ------------------------------------------------------------ CPU oracle leg
def oracle_sample_step(layer, x, W, b, budget_s: float):
    """Times the fp64 CPU oracle on a bounded sample of one step: the full
    quantise + tiled pack of W, and the linear on as many leading token rows
    as fit the time budget.  Returns (extrapolated full-step seconds, rows)."""
    import oracle
    from bit_post_quantised_b200 import workloads

    Wb, xb, bb = workloads.bf16_bits(W), workloads.bf16_bits(x), workloads.bf16_bits(b)
    t0 = time.perf_counter()
    T, s = oracle.quantize(Wb, workloads.EPS)
    oracle.pack_tiled(T)
    t_quant = time.perf_counter() - t0
    rows, t_lin = 0, 0.0
    chunk = max(1, 2 * oracle.num_threads())
    while rows < layer.M and t_lin < budget_s:
        n = min(chunk, layer.M - rows)
        t1 = time.perf_counter()
        oracle.linear(xb[rows:rows + n], T, s, bb)
        t_lin += time.perf_counter() - t1
        rows += n
        chunk = min(chunk * 2, 256)
    return t_quant + t_lin * layer.M / rows, rows, t_quant, t_lin


def cpu_baseline(layer, x, W, b, budget_s: float):
    import oracle

    est, rows, t_quant, t_lin = oracle_sample_step(layer, x, W, b, budget_s)
    return {"value": layer.flop / est / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"full quantise+pack of W [{layer.N},{layer.K}] ({t_quant:.2f} s) and the fp64 "
                       f"linear on {rows} of {layer.M} token rows ({t_lin:.2f} s), extrapolated "
                       f"linearly in rows to the full step ({est:.1f} s)")}


def run_reference(args):
    """--impl reference: the oracle as it stands, on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    if rank != 0:
        return 0
    from bit_post_quantised_b200 import workloads

    layer = workloads.CONFIGS[args.workload]
    x, W, b = workloads.make_inputs(layer)
    per_step = max(0.3, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_step(layer, x, W, b, per_step)
    ests, samples = [], []
    for _ in range(args.steps):
        est, rows, tq, tl = oracle_sample_step(layer, x, W, b, per_step)
        ests.append(est)
        samples.append(rows)
    import oracle

    step_s = statistics.mean(ests)
    value = layer.flop / step_s / 1e12
    sample = (f"each step: full quantise+pack of W and the fp64 linear on the leading "
              f"{min(samples)}-{max(samples)} of {layer.M} token rows, extrapolated to the full step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, FLUX.1-dev QKV shapes)",
        "config": workload_config(layer),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


DESCRIPTIONS = {"qkv": "FLUX.1-dev double-block image-stream QKV, 1024x1024 image",
                "mlp_up": "FLUX.1-dev MLP up projection, 4608 tokens",
                "mlp_down": "FLUX.1-dev MLP down projection, 4608 tokens",
                "tiny": "tiny ternary linear"}


def workload_config(layer, fp8=False):
    what = DESCRIPTIONS.get(layer.name, f"FLUX.1-dev adaLN modulation GEMV ({layer.name})")
    return {"workload": f"{what}: x [{layer.M},{layer.K}] bf16, W [{layer.N},{layer.K}] ternary, bias bf16",
            "M": layer.M, "K": layer.K, "N": layer.N, "eps": 1e-5,
            "step": ("tern_quantize_pack(W) + tern_quantize_act_e4m3(x) + tern_linear_e4m3" if fp8 else
                     "tern_quantize_pack(W) + tern_linear(x)"),
            "accumulate": "fp32",
            "l2": "two rotating input sets of 164 MB each (> 126 MB L2)"}


# ------------------------------------------------------------ GPU arm
def setup_dist(backend: str = "nccl"):
    """Rank layout from the torchrun environment; one process per GPU.  The
    process group (NCCL on GPUs, gloo for the CPU tests of this logic) carries
    only the barriers and the max-over-ranks of the timings: ranks are
    independent replicas with no collective on the data path."""
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def _collective_device():
    import torch
    import torch.distributed as dist

    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier(world):
    import torch

    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def max_over_ranks(value: float, world: int) -> float:
    """Largest of the ranks' values (every rank gets it): a multi-GPU time is
    the slowest rank's."""
    import torch

    if world == 1:
        return value
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=_collective_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, flop_per_step: float, elapsed_s: float) -> float:
    """Whole-job TFLOP/s: every rank ran `steps` steps of `flop_per_step`
    within `elapsed_s` (the max over ranks)."""
    return world * steps * flop_per_step / elapsed_s / 1e12


def make_sets(layer, rank, n_sets, device):
    """Per-rank input sets (rank-dependent seeds: independent replicas)."""
    import dataclasses

    import torch

    from bit_post_quantised_b200 import workloads

    sets = []
    for i in range(n_sets):
        L = dataclasses.replace(layer, seed=layer.seed + 7919 * rank + 104729 * i)
        x, W, b = workloads.make_inputs(L)
        sets.append({
            "x": x.to(device), "W": W.to(device), "b": b.to(device),
            "packed": torch.empty(layer.N * layer.K // 4, dtype=torch.uint8, device=device),
            "scales": torch.empty(layer.N, dtype=torch.float32, device=device),
            "y": torch.empty(layer.M, layer.N, dtype=torch.bfloat16, device=device),
            "xq": torch.empty(layer.M, layer.K, dtype=torch.uint8, device=device),
            "a": torch.empty(layer.M, dtype=torch.float32, device=device),
            "cpu": (x, W, b),
        })
    return sets


def graph_time(calls, replays, stream):
    """Device time per call of a list of launches captured in one CUDA graph
    (removes host launch overhead from microsecond kernels)."""
    import torch

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for c in calls:  # warm-up on the capture stream (allocates its workspace)
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(replays):
            g.replay()
    e1.record(stream)
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e-3 / (replays * len(calls))


def interleaved_time(call_lists, rounds, stream):
    """Device time per call of several launch lists, each captured in its own
    CUDA graph, replayed in turn round after round (median over rounds).
    Under the power cap the SM clock drifts over tens of milliseconds, so
    cases timed one after another see different clocks; taking turns gives
    every case the same mix of them (a fused epilogue is compared with the
    plain layer this way)."""
    import statistics

    import torch

    graphs = []
    for calls in call_lists:
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for c in calls:  # warm-up on the capture stream
                c()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in calls:
                c()
        graphs.append(g)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    times = [[] for _ in graphs]
    for _ in range(rounds):
        for i, g in enumerate(graphs):
            e0.record(stream)
            with torch.cuda.stream(stream):
                g.replay()
            e1.record(stream)
            e1.synchronize()
            times[i].append(e0.elapsed_time(e1) * 1e-3 / len(call_lists[i]))
    del graphs
    return [statistics.median(t) for t in times]


def cublas_context_us(L, packs, x, b, stream):
    """Dense bf16 cuBLAS (F.linear) on the dequantised weight T*s of the same
    shape, as context: the weight rotates over enough copies (> 3x the 126 MB
    L2) that it is read from HBM, like the ternary codes."""
    import torch
    import torch.nn.functional as F

    from bit_post_quantised_b200 import tern

    l2 = 126 * 2 ** 20
    wbytes = 2 * L.N * L.K
    copies = max(2, min(len(packs), -(-3 * l2 // wbytes) + 1))
    Wds = [tern.dequantize(packs[i % len(packs)][0], packs[i % len(packs)][1], L.K, stream=stream)
           for i in range(copies)]
    torch.cuda.synchronize()
    reps = max(2, 24 // copies)
    t = graph_time([(lambda Wd=Wd: F.linear(x, Wd, b)) for Wd in Wds] * reps, 5, stream)
    del Wds
    return t * 1e6


def side_table(device, peaks, stream):
    """Per-kernel figures for the other rows of the path (not the headline):
    the adaLN modulation GEMV sweep, the MLP layers, quantise/pack, the adaLN
    modulation of normalised activations, and bf16 cuBLAS on the dequantised
    weight (torch's unfused normalisation for the latter) as context.  Weights rotate over enough
    copies that they do not stay in L2 between launches."""
    import torch
    import torch.nn.functional as F

    from bit_post_quantised_b200 import tern, workloads

    rows = {}
    l2 = 126 * 2 ** 20
    for name in ["mod6_m1", "mod6_m4", "mod6_m16", "mod6_m64", "mod3_m1", "mod3_m4", "mod3_m16",
                 "mod3_m64", "qkv", "mlp_up", "mlp_down"]:
        L = workloads.CONFIGS[name]
        x, W, b = (t.to(device) for t in workloads.make_inputs(L))
        copies = max(2, min(24, int(3 * l2 // max(1, L.packed_bytes)) + 1))
        packs = []
        for _ in range(copies):
            packs.append(tern.quantize_pack(W, workloads.EPS, stream=stream))
        y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=device)
        calls = [(lambda p=p, s=s: tern.linear(x, p, s, b, out=y)) for p, s in packs]
        reps = max(2, 64 // copies)
        fused = None
        if name == "mlp_up":
            # FLUX's MLP activation fused into the epilogue
            fused = [(lambda p=p, s=s: tern.linear_act(x, p, s, b, tern.ACT_GELU_TANH, 0, out=y)) for p, s in packs]
        elif name == "qkv":
            # per-head RMS normalisation of q and k (the first 2 * HIDDEN
            # columns) fused into the epilogue
            nw = (1 + 0.1 * torch.randn(L.N, device=device)).to(torch.bfloat16)
            fused = [(lambda p=p, s=s: tern.linear_epilogue(x, p, s, b, norm_cols=(0, 2 * workloads.HIDDEN),
                                                            norm_weight=nw, norm_eps=1e-6, out=y))
                     for p, s in packs]
            # and the rotary embedding of the image tokens' positions (0, row,
            # column) on the 64 x 64 grid after the normalisation
            from bit_post_quantised_b200 import flux
            side = int(round(L.M ** 0.5))
            ids = torch.zeros(L.M, 3, dtype=torch.float64)
            ids[:, 1] = torch.arange(L.M, dtype=torch.float64) // side
            ids[:, 2] = torch.arange(L.M, dtype=torch.float64) % side
            cs = torch.stack(flux.rope_cos_sin(ids), dim=-1).contiguous().to(device)
            roped = [(lambda p=p, s=s: tern.linear_epilogue(x, p, s, b, norm_cols=(0, 2 * workloads.HIDDEN),
                                                            norm_weight=nw, norm_eps=1e-6, rope_cs=cs, out=y))
                     for p, s in packs]
        if fused is None:
            t = graph_time(calls * reps, 5, stream)
        elif name == "qkv":
            t, tf, tr = interleaved_time([c * (reps // 2 or 1) for c in (calls, fused, roped)], 8, stream)
        else:
            t, tf = interleaved_time([calls * (reps // 2 or 1), fused * (reps // 2 or 1)], 8, stream)
        flop_t = 2.0 * L.M * L.N * L.K / peaks["bf16_tflops"] / 1e12
        byte_t = L.algorithmic_bytes / peaks["hbm_gbs"] / 1e9
        entry = {"M": L.M, "N": L.N, "K": L.K, "us": t * 1e6, "tflops": L.flop / t / 1e12,
                 "packed_gbs": L.packed_bytes / t / 1e9, "roofline_frac": max(flop_t, byte_t) / t,
                 "bound": "tensor" if flop_t > byte_t else "hbm"}
        if name == "mlp_up":
            # against the HBM time a separate bf16 GELU pass over y would
            # need (read + write); plain and fused timed in turns
            entry["gelu_fused_us"] = tf * 1e6
            entry["gelu_separate_pass_us_at_hbm_peak"] = 2 * 2 * L.M * L.N / peaks["hbm_gbs"] / 1e9 * 1e6
        elif name == "qkv":
            # against the HBM time a separate pass over q and k would need
            entry["qk_norm_fused_us"] = tf * 1e6
            entry["qk_norm_rope_fused_us"] = tr * 1e6
            entry["qk_norm_separate_pass_us_at_hbm_peak"] = (2 * 2 * L.M * 2 * workloads.HIDDEN / peaks["hbm_gbs"]
                                                              / 1e9 * 1e6)
        entry["cublas_bf16_us"] = cublas_context_us(L, packs, x, b, stream)
        rows[name] = entry
        del packs
    # FP8 (E4M3) activations on the QKV shape: the per-token quantisation of x
    # and the kind::f8f6f4 layer, against the FP8 tensor peak (the measured
    # bf16 burst x 2, the nominal dense ratio)
    L = workloads.CONFIGS["qkv"]
    x, W, b = (t.to(device) for t in workloads.make_inputs(L))
    packs = [tern.quantize_pack(W, workloads.EPS, stream=stream) for _ in range(24)]
    xq, a = tern.quantize_act_e4m3(x, stream=stream)
    y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=device)
    t_lin = graph_time([(lambda p=p, s=s: tern.linear_e4m3(xq, a, p, s, b, out=y, stream=stream))
                        for p, s in packs] * 2, 5, stream)
    xs4 = [(torch.randn(L.M, L.K, device=device)).to(torch.bfloat16) for _ in range(6)]  # 151 MB > L2
    t_q = graph_time([(lambda xx=xx: tern.quantize_act_e4m3(xx, xq=xq, a=a, stream=stream)) for xx in xs4] * 4, 5,
                     stream)
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    qbytes = 2 * L.M * L.K + L.M * L.K + 4 * L.M
    rows["qkv_fp8_activations"] = {
        "M": L.M, "N": L.N, "K": L.K, "linear_us": t_lin * 1e6, "tflops": L.flop / t_lin / 1e12,
        "fp8_peak_tflops": fp8_peak, "frac_of_fp8_peak": L.flop / t_lin / 1e12 / fp8_peak,
        "peak_source": "measured bf16 burst x 2 (nominal dense FP8/BF16 ratio)",
        "quantize_act_us": t_q * 1e6, "quantize_act_gbs": qbytes / t_q / 1e9,
        "quantize_act_hbm_frac": qbytes / t_q / 1e9 / peaks["hbm_gbs"],
        "step_us": (t_lin + t_q) * 1e6, "step_tflops": L.flop / (t_lin + t_q) / 1e12}
    del packs, xs4, xq, a, y
    # quantise/pack of the largest weight
    N, K = 21504, 3072
    W = (torch.randn(N, K, device=device) * 0.02).to(torch.bfloat16)
    p = torch.empty(N * K // 4, dtype=torch.uint8, device=device)
    s = torch.empty(N, dtype=torch.float32, device=device)
    t = graph_time([lambda: tern.quantize_pack(W, packed=p, scales=s)] * 10, 5, stream)
    nbytes = 2 * N * K + N * K // 4 + 4 * N
    rows["quantize_pack_21504x3072"] = {"us": t * 1e6, "gbs": nbytes / t / 1e9,
                                        "hbm_frac": nbytes / t / 1e9 / peaks["hbm_gbs"]}
    del W, p, s
    # adaLN modulation of a single block's 4608 token rows (one image), four
    # x/out pairs rotating (226 MB > L2); torch's unfused layer_norm, multiply
    # and add as context
    M, K = 4608, 3072
    mod = (torch.randn(1, 6 * K, device=device) * 0.1).to(torch.bfloat16)
    xs_ = [(torch.randn(M, K, device=device)).to(torch.bfloat16) for _ in range(4)]
    outs_ = [torch.empty_like(xs_[0]) for _ in range(4)]
    calls = [(lambda x=x, o=o: tern.adaln_modulate(x, mod[:, K:2 * K], mod[:, :K], 1e-6, out=o))
             for x, o in zip(xs_, outs_)]
    t = graph_time(calls * 3, 5, stream)
    nbytes = 2 * 2 * M * K + 2 * 2 * K
    sc_, sh_ = mod[0, K:2 * K], mod[0, :K]
    tu = graph_time([(lambda x=x: F.layer_norm(x, (K,), eps=1e-6) * (1 + sc_) + sh_) for x in xs_] * 3, 5, stream)
    rows["adaln_modulate_4608x3072"] = {"us": t * 1e6, "gbs": nbytes / t / 1e9,
                                        "hbm_frac": nbytes / t / 1e9 / peaks["hbm_gbs"],
                                        "torch_unfused_us": tu * 1e6}
    del xs_, outs_, mod
    rows.update(stack_rows(device, peaks, stream))
    rows.update(forward_rows(device, peaks, stream))
    return rows


def stack_rows(device, peaks, stream):
    """The whole ternary linear stack of one FLUX.1-dev forward at 1024x1024
    (19 double + 38 single blocks; weights drawn on the device from N(0, 0.02)
    per layer seed and quantised, only the codes kept), run block by block
    through tern_linear_batch_epilogue with synthetic activations, the MLP's
    GELU fused into its first linear (the MLP columns of a single block's
    fused projection) and the gated residual update fused into the output
    projections, and the 76 adaLN modulation GEMVs of a forward alone:
    batched versus one call each."""
    import torch

    from bit_post_quantised_b200 import tern, workloads

    layers = workloads.flux_stack()
    packs = []
    for L in layers:
        g = torch.Generator(device=device).manual_seed(L.seed)
        W = (torch.randn(L.N, L.K, generator=g, device=device) * L.w_std).to(torch.bfloat16)
        packs.append(tern.quantize_pack(W, workloads.EPS, stream=stream))
        del W
    bias = {}
    xs, ys = {}, {}

    def buf(d, key, shape):
        if key not in d:
            d[key] = (torch.randn(*shape, device=device) * 0.5).to(torch.bfloat16)
        return d[key]

    blocks = {}
    for i, L in enumerate(layers):
        blocks.setdefault(L.name.split(".")[0], []).append(i)
    problems = []  # per block: list of dicts for tern_linear_batch
    for name, idx in blocks.items():
        probs = []
        for j, i in enumerate(idx):
            L = layers[i]
            if L.N not in bias:
                bias[L.N] = (torch.randn(L.N, device=device) * 0.01).to(torch.bfloat16)
            p = dict(x=buf(xs, (L.M, L.K), (L.M, L.K)), packed=packs[i][0], scales=packs[i][1], bias=bias[L.N],
                     y=buf(ys, (j, L.M, L.N), (L.M, L.N)))
            e = workloads.block_epilogue(L.name)
            if e.get("act") == "gelu_tanh":
                p["act"], p["act_col0"] = tern.ACT_GELU_TANH, e["act_col0"]
            elif e.get("gated_residual"):
                # gated update of a residual stream, in place (adaLN-Zero); one
                # buffer per problem, as the problems of a batch run concurrently
                stream_buf = buf(ys, ("stream", j, L.M, L.N), (L.M, L.N))
                p["y"], p["residual"] = stream_buf, stream_buf
                p["gate"] = buf(xs, ("gate", L.N), (L.N,))
            probs.append(p)
        problems.append(probs)
    flop = sum(L.flop for L in layers)

    def forward():
        for probs in problems:
            tern.linear_batch_epilogue(probs, stream=stream)

    t = graph_time([forward], 3, stream)
    out = {"flux_stack": {"layers": len(layers), "launch_groups": "one tern_linear_batch_epilogue per block",
                          "epilogue": ("GELU (tanh form) fused into every MLP up projection; gated in-place "
                                       "residual update fused into every attention/MLP output projection"),
                          "ms_per_forward": t * 1e3, "tflops": flop / t / 1e12,
                          "tensor_roofline_ms": flop / (peaks["bf16_tflops"] * 1e12) * 1e3,
                          "packed_weight_gb": sum(L.packed_bytes for L in layers) / 1e9}}
    mods = [dict(x=buf(xs, (1, L.K), (1, L.K)), packed=packs[i][0], scales=packs[i][1], bias=bias[L.N],
                 y=buf(ys, ("mod", i), (1, L.N))) for i, L in enumerate(layers) if L.name.endswith(".mod")]
    mod_bytes = sum(p["packed"].numel() for p in mods)
    t_batch = graph_time([lambda: tern.linear_batch(mods, stream=stream)], 5, stream)
    t_each = graph_time([lambda: [tern.linear(p["x"], p["packed"], p["scales"], p["bias"], out=p["y"],
                                              stream=stream) for p in mods]], 5, stream)
    out["modulation_gemvs_per_forward"] = {
        "count": len(mods), "packed_mb": mod_bytes / 1e6,
        "batched_us": t_batch * 1e6, "batched_packed_gbs": mod_bytes / t_batch / 1e9,
        "one_call_each_us": t_each * 1e6, "hbm_frac_batched": mod_bytes / t_batch / 1e9 / peaks["hbm_gbs"]}
    return out


def forward_rows(device, peaks, stream):
    """A FLUX.1-shaped forward at 1024x1024 (19 double + 38 single blocks,
    seeded random weights, synthetic inputs): the unquantised input layers
    and embedders and the final layer in bf16 (cuBLAS), every block linear
    ternary through the library with its fused epilogues (the rotary
    embedding in the q/k epilogue), attention from torch; against the same
    model with the blocks in bf16 with dense weights (T*s) through cuBLAS and
    torch's unfused operations, the bf16 model of the pages' Table 3
    comparison.  The two are timed in turns (CUDA events, medians of 3),
    launched from Python and replayed from CUDA graphs."""
    import statistics

    import torch

    from bit_post_quantised_b200 import flux, workloads

    cfg = workloads.FluxConfig()
    model = flux.TernaryFlux(cfg, device=device)
    io = {k: (W.to(device), b.to(device)) for k, (W, b) in workloads.flux_io_weights(cfg).items()}
    img, txt, pooled, t, g, ids = workloads.flux_model_inputs(cfg)
    args = (img.to(device), txt.to(device), pooled.to(device), t, g, ids.to(device))
    dense = flux.dense_weights(model)
    runs = {"ternary": lambda: flux.model_forward(model, io, *args),
            "dense_bf16": lambda: flux.dense_model_forward(model, dense, io, *args)}
    for f in runs.values():
        f()
    torch.cuda.synchronize()
    # the same forwards replayed from CUDA graphs (no host launch gaps)
    graphs = {}
    side = torch.cuda.Stream(device)
    for k, f in list(runs.items()):
        side.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(side):
            f()
        torch.cuda.current_stream(device).wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            f()
        graphs[k] = g
        runs[k + "_graph"] = g.replay
    for k in ("ternary_graph", "dense_bf16_graph"):
        runs[k]()
    torch.cuda.synchronize()
    times = {k: [] for k in runs}
    for _ in range(3):
        for k, f in runs.items():
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            e1.synchronize()
            times[k].append(e0.elapsed_time(e1))
    fl = flux.forward_flop(cfg)
    packed = sum(q[n][0].numel() for q in model.blocks.values() for n in q if not n.endswith("norm_w"))
    dense_b = sum(d[n][0].numel() * 2 for d in dense.values() for n in d if not n.endswith("norm_w"))
    io_b = sum(W.numel() * 2 for W, _ in io.values())
    t_ter, t_den = statistics.median(times["ternary"]), statistics.median(times["dense_bf16"])
    tg_ter, tg_den = statistics.median(times["ternary_graph"]), statistics.median(times["dense_bf16_graph"])
    del graphs, runs, dense, model
    torch.cuda.empty_cache()
    return {"flux_forward": {
        "model": f"{cfg.n_double} double + {cfg.n_single} single blocks, {cfg.img_tokens} image + "
                 f"{cfg.txt_tokens} text tokens, input layers, embedders and final layer",
        "ternary_ms": t_ter, "dense_bf16_ms": t_den, "speedup_vs_dense_bf16": t_den / t_ter,
        "ternary_graph_ms": tg_ter, "dense_bf16_graph_ms": tg_den, "speedup_graph": tg_den / tg_ter,
        "linear_gflop": fl["linear"] / 1e9, "attention_gflop": fl["attention"] / 1e9,
        "ternary_tflops": (fl["linear"] + fl["attention"]) / (t_ter * 1e-3) / 1e12,
        "block_weight_gb_ternary": packed / 1e9, "block_weight_gb_bf16": dense_b / 1e9,
        "io_layer_weight_gb_bf16": io_b / 1e9,
        "outside": "attention (torch SDPA), SiLU and the unquantised input/output layers (bf16 cuBLAS): torch; "
                   "all block linears (with q/k norm and rotary embedding, GELU, gated residual in their "
                   "epilogues) and the adaLN passes: this library"}}


def gpu_id_for_smi(local: int) -> str:
    """nvidia-smi --id for the CUDA device (by UUID, so visible-device
    remapping cannot point the sampler at another GPU)."""
    import torch

    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


def run_tern(args):
    import torch

    from bit_post_quantised_b200 import tern, workloads

    world, rank, local = setup_dist("nccl")
    device = torch.device("cuda", local)
    stream = torch.cuda.Stream(device)
    peaks = load_peaks()
    layer = workloads.CONFIGS[args.workload]
    sets = make_sets(layer, rank, 2, device)
    K, Wm = args.steps, max(3, args.warmup)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    def layer_call(st):
        if args.fp8:
            tern.quantize_act_e4m3(st["x"], xq=st["xq"], a=st["a"], stream=stream)
            tern.linear_e4m3(st["xq"], st["a"], st["packed"], st["scales"], st["b"], out=st["y"], stream=stream)
        else:
            tern.linear(st["x"], st["packed"], st["scales"], st["b"], out=st["y"], stream=stream)

    def step(i, events=None):
        st = sets[i % len(sets)]
        if events:
            events[0].record(stream)
        tern.quantize_pack(st["W"], workloads.EPS, packed=st["packed"], scales=st["scales"], stream=stream)
        if args.fp8:
            tern.quantize_act_e4m3(st["x"], xq=st["xq"], a=st["a"], stream=stream)
        if events:
            events[1].record(stream)
        if args.fp8:
            tern.linear_e4m3(st["xq"], st["a"], st["packed"], st["scales"], st["b"], out=st["y"], stream=stream)
        else:
            tern.linear(st["x"], st["packed"], st["scales"], st["b"], out=st["y"], stream=stream)
        if events:
            events[2].record(stream)

    for i in range(Wm):
        step(i)
    barrier(world)
    if tern.device_status(stream) != 0:
        raise RuntimeError("device wait timed out during warm-up")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id_for_smi(local)) as clocks:
        barrier(world)
        t0.record(stream)
        for i in range(K):
            step(i, ev[i])
        t1.record(stream)
        t1.synchronize()
        barrier(world)
    elapsed = max_over_ranks(t0.elapsed_time(t1) * 1e-3, world)
    if tern.device_status(stream) != 0:
        raise RuntimeError("device wait timed out during the timed steps")
    t_quant = statistics.mean(e[0].elapsed_time(e[1]) for e in ev) * 1e-3
    t_lin = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) * 1e-3
    t_lin = max_over_ranks(t_lin, world)

    # ---- end to end through the public API, from pinned host buffers
    host = []
    for st in sets:
        x, W, b = st["cpu"]
        host.append({"x": x.pin_memory(), "W": W.pin_memory(), "b": b.pin_memory(),
                     "y": torch.empty(layer.M, layer.N, dtype=torch.bfloat16).pin_memory()})
    h2d = sum(host[0][k].numel() * host[0][k].element_size() for k in ("x", "W", "b"))
    d2h = host[0]["y"].numel() * host[0]["y"].element_size()

    # Three streams so that step i's inputs cross PCIe (host->device) while
    # step i-1 computes and step i-2's y comes back (PCIe is full duplex).
    # Every step still copies its own inputs in and its y out inside the
    # timed region; events keep each device set's reuse in order.
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    nset = len(sets)
    ev_in = [torch.cuda.Event() for _ in range(nset)]
    ev_comp = [torch.cuda.Event() for _ in range(nset)]
    ev_out = [torch.cuda.Event() for _ in range(nset)]
    used = [False] * nset

    def e2e_step(i):
        j = i % nset
        st, hs = sets[j], host[j]
        if used[j]:
            s_in.wait_event(ev_comp[j])  # step i - nset no longer reads this set's inputs
        with torch.cuda.stream(s_in):
            st["W"].copy_(hs["W"], non_blocking=True)
            st["x"].copy_(hs["x"], non_blocking=True)
            st["b"].copy_(hs["b"], non_blocking=True)
        ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if used[j]:
            stream.wait_event(ev_out[j])  # step i - nset's y has left the device
        tern.quantize_pack(st["W"], workloads.EPS, packed=st["packed"], scales=st["scales"], stream=stream)
        layer_call(st)
        ev_comp[j].record(stream)
        s_out.wait_event(ev_comp[j])
        with torch.cuda.stream(s_out):
            hs["y"].copy_(st["y"], non_blocking=True)
        ev_out[j].record(s_out)
        used[j] = True

    def e2e_run(n):
        t0.record(s_in)
        stream.wait_event(t0)
        s_out.wait_event(t0)
        for i in range(n):
            e2e_step(i)
        stream.wait_event(ev_out[(n - 1) % nset])
        s_in.wait_event(ev_out[(n - 1) % nset])
        for j in range(nset):
            s_out.wait_event(ev_comp[j])
        t1.record(s_out)
        t1.synchronize()

    e2e_run(Wm)
    barrier(world)
    e2e_run(K)
    barrier(world)
    e2e_elapsed = max_over_ranks(t0.elapsed_time(t1) * 1e-3, world)

    flop = layer.flop
    value = job_throughput(world, K, flop, elapsed)
    achieved = flop / t_lin / 1e12
    tensor_bound = flop / (peaks["bf16_tflops"] * 1e12) >= layer.algorithmic_bytes / (peaks["hbm_gbs"] * 1e9)
    kname, kstem = linear_kernel(layer)
    traffic = profiled_traffic(kstem, layer.name)
    if args.fp8:
        # FP8 tensor peak: the measured bf16 burst x 2 (the nominal dense ratio)
        peaks = dict(peaks, bf16_tflops=2.0 * peaks["bf16_tflops"], source=peaks["source"] + " bf16 x 2 (FP8)")
        kname, kstem = "ternary_fp8_pair_kernel", "ternary_fp8"
        traffic = profiled_traffic(kstem, layer.name)
        tensor_bound = True
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": elapsed / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 x, ternary w" if args.fp8 else "bf16",
        "data": "synthetic (seeded, FLUX.1-dev QKV shapes)",
        "config": workload_config(layer, args.fp8),
        "roofline": ({"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                      "kernel": f"{kname} ({'tern_linear_e4m3' if args.fp8 else 'tern_linear'})",
                      "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)"}
                     if tensor_bound else
                     {"bound": "hbm", "achieved": layer.algorithmic_bytes / t_lin / 1e9,
                      "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": layer.algorithmic_bytes / t_lin / 1e9 / peaks["hbm_gbs"], "traffic": traffic,
                      "kernel": f"{kname} (tern_linear)",
                      "peak_source": f"{peaks['source']} HBM copy (MEASURED_PEAKS.json)"}),
        "linear_us": t_lin * 1e6, "quantize_pack_us": t_quant * 1e6,
        "packed_weight_gbs": layer.packed_bytes / t_lin / 1e9,
        "quantize_pack_gbs": (2 * layer.N * layer.K + layer.packed_bytes + 4 * layer.N) / t_quant / 1e9,
        "e2e": {"value": job_throughput(world, K, flop, e2e_elapsed), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (3 if args.fp8 else 2) * K * world,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and args.cpu_seconds > 0 and not args.fp8:
        line["cpu_baseline"] = cpu_baseline(layer, *sets[0]["cpu"], budget_s=args.cpu_seconds)
        if not args.no_extras:
            try:
                line["side_table"] = side_table(device, peaks, stream)
            except Exception as e:  # the side table is context; never lose the main line
                line["side_table"] = {"error": f"{type(e).__name__}: {e}"}
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_tern(args)


if __name__ == "__main__":
    sys.exit(main())
