"""Benchmark of the INT8 ConvRot linear layer on B200: one JSON line on stdout.

A step is one full ConvRot linear call (rotate + per-token quantise, int8 GEMM
on tcgen05, dequantise + bias) through the C ABI on one batch of synthetic
input already resident in HBM. The default workload is the DiT fused-QKV
projection at 1024^2: M=4608 tokens (4096 image + 512 text), K=3072, N=9216,
g=256, with bias.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm
    python bench.py --dtype f16 --wscale channel --act gelu   # a layer variant (convrot_linear_ex)

Besides the headline the line carries:
  * ``int8_peak``: the int8 tensor pipe's rate measured on this GPU by a probe
    that issues the GEMM's own instruction (tcgen05.mma.cta_group::2.kind::i8,
    256x256x32) from shared memory with no global traffic, in bursts and in a
    longer loop under the power limit (sustained), on zero operands and on
    operand tiles copied from the layer's own codes. The tensor cores draw more
    power on real codes and the GPU lowers its clock sooner, so the rate on the
    codes (the larger of its burst and sustained figures) is the GEMM's roofline
    denominator; the zero-operand rate and the fraction against it are reported
    beside it;
  * ``configs``: every layer shape of the workload table timed by CUDA events
    (median and min over the repetitions, inputs rotated over enough buffer
    sets to exceed L2): the layer's time per call, TOPS, the GEMM's TOPS and
    fraction of the int8 peak, the rotate+quantise pass's GB/s and fraction of
    HBM, and for the weight-streaming shapes (M <= 128) the fraction of HBM on
    the layer's algorithmic bytes;
  * ``e2e``: the same metric through the public Python API with host buffers,
    the host-to-device copies, the layers and the device-to-host copies on
    three streams ordered by events over the rotating buffer sets.

Under torchrun (N > 1) every rank runs an independent replica of the same
workload on its own GPU (the layer has no cross-GPU step); the value is the
work of all ranks over the slowest rank's device time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ConvRot linear TOPS (rotate+quant+i8 GEMM+dequant) and % of B200 INT8 peak"
UNIT = "TOPS"
N_SETS = 4  # rotating input/output sets per rank so that no step finds its data in L2
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 4.5 / 2.25  # nominal dense int8 : dense bf16 tensor rate on B200 (context only)
NOMINAL_INT8_TOPS = 4500.0  # datasheet dense int8 (context only)
WS_CLOCK_RECORD_OFFSET = 64  # CONVROT_WS_CLOCK_RECORD_OFFSET in include/convrot.h
PEAK_BURST_REGION_MS = 50.0
IDLE_BEFORE_REGION_S = 0.5  # idle time before the per-launch timed region
WARMUP_AFTER_IDLE = 30  # untimed steps between that idle time and the region  # timed regions up to this long are compared with the probe's burst rate
SMALL_M = 64  # up to this many tokens the layer's GEMM is the weight-streaming form
PROBE_OPS_PER_ITER_PER_PAIR = 2.0 * 256 * 256 * 128  # four 256x256x32 MMAs

# DRAM bytes per launch of the dominant kernel (the pair GEMM) on a workload,
# from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum). A
# figure holds only for the kernel source it was taken on: the sha256 over
# GEMM_SOURCES (the files the pair kernel is compiled from) must match,
# otherwise the bench reports null.
GEMM_SOURCES = ["gemm_i8.cu", "gemm_i8.cuh", "ptx_sm100.cuh"]
GEMM_TRAFFIC = {
    "dit_qkv_1024": {"bytes": 42703616 + 41476608,
                     "sources_sha256": "4c38e302f0c1937c269bdc42ceec44889b1300d216684d7c326b53e8b97befb2"},
}

# Every layer shape of the workload table, timed after the headline.
CONFIG_NAMES = ["tiny", "dit_qkv_1024", "dit_mlp_up_1024", "dit_mlp_down_1024", "dit_mlp_2048",
                "textenc_m1", "textenc_m16", "textenc_m128", "textenc_m512"]


def gemm_traffic(config: str):
    import hashlib

    rec = GEMM_TRAFFIC.get(config)
    if rec is None:
        return None
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "w8a8_rotated_int8_token_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return float(rec["bytes"]) if h.hexdigest() == rec["sources_sha256"] else None


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="dit_qkv_1024")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config table")
    ap.add_argument("--no-peak", action="store_true", help="skip the int8 peak probe")
    ap.add_argument("--config-reps", type=int, default=30, help="timed repetitions per config")
    ap.add_argument("--attention-only", action="store_true",
                    help="time only the INT8 attention call (--config-reps calls) and print its figures")
    # layer variants (convrot_linear_ex); the defaults are the headline layer
    ap.add_argument("--dtype", choices=["bf16", "f16"], default="bf16", help="dtype of X, W, bias and Y")
    ap.add_argument("--wscale", choices=["tensor", "channel"], default="tensor", help="weight-scale granularity")
    ap.add_argument("--act", choices=["none", "gelu"], default="none", help="activation fused into the epilogue")
    return ap.parse_args(argv)


def reduce_max(v: float, device) -> float:
    """The maximum of v over the ranks of the default process group (v itself
    with one rank): every multi-rank time is the slowest rank's."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(ops_per_step: float, steps: int, world: int, t_ms: float) -> float:
    """Whole-job throughput: the work of all ranks over the (max-over-ranks) time."""
    return ops_per_step * steps * world / (t_ms * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w) -> dict:
    return {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "g": w.g, "bias": w.bias,
            "x": f"{w.x_dist}, {w.outlier_frac:g} outlier channels x{w.outlier_mult:g}",
            "w_std": w.w_std,
            "l2": f"{N_SETS} rotating input/output sets per GPU, each step on a set last used "
                  f"{N_SETS - 1} steps earlier (>126 MB L2 in between)"}


def sets_for(bytes_per_set: float) -> int:
    """Rotating buffer sets so that a set is reused only after more than L2's worth of other sets."""
    return int(min(8, max(N_SETS, math.ceil(2 * L2_BYTES / max(bytes_per_set, 1.0)) + 1)))


def med_min(xs):
    return float(statistics.median(xs)), float(min(xs))


# --------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running (read only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------- CPU oracle


def cpu_oracle_leg(d, target_s: float, gpu_y=None):
    """Time the oracle (as it stands) on a bounded sample of the workload.

    The sample is the first `rows` tokens (all of them when a full pass takes
    less than the target), repeated until about `target_s` seconds of CPU work.
    """
    import oracle
    from threadpoolctl import threadpool_info

    w = d["workload"]
    x = oracle.bf16_to_f64(d["x"])
    wf = oracle.bf16_to_f64(d["w"])
    b = None if d["bias"] is None else oracle.bf16_to_f64(d["bias"])
    wq, sw = oracle.prepare_weight(wf, w.g)  # once per layer, untimed like the GPU side
    rows = min(64, w.M)
    t0 = time.perf_counter()
    oracle.linear(x[:rows], wq, sw, w.g, b)
    t1 = max(time.perf_counter() - t0, 1e-3)
    rows = int(max(1, min(w.M, rows * target_s / t1)))
    reps, dt, y = 0, 0.0, None
    while reps == 0 or (dt < target_s and reps < 100):
        t0 = time.perf_counter()
        y = oracle.linear(x[:rows], wq, sw, w.g, b)
        dt += time.perf_counter() - t0
        reps += 1
    threads = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
    cores = int(max(threads)) if threads else os.cpu_count()
    tops = 2.0 * rows * w.N * w.K * reps / dt / 1e12
    parity = None
    if gpu_y is not None:
        parity = oracle.nrmse(gpu_y[:rows], y)
    return {"value": tops, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{reps} x the first {rows} of {w.M} tokens of {w.name} through the float64 oracle "
                      f"(rotate, quantise, GEMM, dequantise; weight prepared beforehand), {dt:.1f} s"}, parity


def run_reference(args):
    """Reference arm: the CPU oracle, rank 0 only, bounded samples."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth

    d = synth.make_workload(args.config)
    w = d["workload"]
    import oracle

    x = oracle.bf16_to_f64(d["x"])
    b = None if d["bias"] is None else oracle.bf16_to_f64(d["bias"])
    wq, sw = oracle.prepare_weight(oracle.bf16_to_f64(d["w"]), w.g)
    total_budget = 150.0  # seconds for warm-up + timed steps
    rows = min(8, w.M)
    t0 = time.perf_counter()
    oracle.linear(x[:rows], wq, sw, w.g, b)
    t_one = max(time.perf_counter() - t0, 1e-3)
    per_step = total_budget / max(1, args.steps + args.warmup)
    rows = int(max(1, min(w.M, rows * per_step / t_one)))
    for i in range(args.warmup):
        oracle.linear(x[:rows], wq, sw, w.g, b)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.linear(x[:rows], wq, sw, w.g, b)
    dt = time.perf_counter() - t0
    from threadpoolctl import threadpool_info

    threads = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
    cores = int(max(threads)) if threads else os.cpu_count()
    value = 2.0 * rows * w.N * w.K * args.steps / dt / 1e12
    sample = f"first {rows} of {w.M} tokens of {w.name} per step through the float64 CPU oracle"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


# ------------------------------------------------------------------ GPU


def bits_to_dev(bits, dev, dtype=None):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    return t if dtype is None or dtype == torch.bfloat16 else t.to(dtype)


def measure_i8_peak(cr, dev, stream, clock_index: int, burst_ms: float = 5.0, sustained_s: float = 0.4,
                    operands=None) -> dict:
    """The int8 tensor pipe's rate on this GPU (probe of the GEMM's own instruction, no global traffic).

    burst: single launches of about `burst_ms`, timed by events, after two warm-up
    launches (the GEMM is timed the same way, alone or inside short steps);
    sustained: launches back to back for about `sustained_s` under the power limit.
    With `operands` (the layer's own codes) the same two figures are taken again on
    them: the tensor cores draw more power on real codes than on zeros, and the GPU
    lowers its clock under its power limit sooner.
    """
    import torch

    ws = torch.empty((256,), dtype=torch.uint8, device=dev)
    r = _probe_i8_rates(cr, dev, stream, clock_index, ws, None, burst_ms, sustained_s)
    if operands is not None:
        c = _probe_i8_rates(cr, dev, stream, clock_index, ws, operands, burst_ms, sustained_s)
        r["on_layer_codes"] = {k: c[k] for k in ("burst_tops", "burst_tops_median", "sustained_tops",
                                                 "burst_clock_mhz", "sustained_clock_mhz", "reasons",
                                                 "burst_sm_mhz_in_kernel", "sustained_sm_mhz_in_kernel",
                                                 "ops_per_clk_per_sm_in_kernel")}
    return r


def kernel_clock_mhz(ws) -> float | None:
    """The SM clock a GEMM or probe launch ran at, from the clock record it left in its workspace
    (%clock64 and %globaltimer twice; include/convrot.h, CONVROT_WS_CLOCK_RECORD_OFFSET)."""
    import torch

    rec = ws[WS_CLOCK_RECORD_OFFSET:WS_CLOCK_RECORD_OFFSET + 32].view(torch.int64).tolist()
    dc, dt = rec[2] - rec[0], rec[3] - rec[1]
    return dc / dt * 1e3 if dc > 0 and dt > 0 else None


def _probe_i8_rates(cr, dev, stream, clock_index: int, ws, operands, burst_ms: float, sustained_s: float) -> dict:
    import torch

    ctas = cr.convrot_probe_i8_peak(64, operands=operands, ws=ws, stream=stream)
    torch.cuda.synchronize(dev)
    pairs = ctas // 2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # calibrate the iteration count to about burst_ms per launch
    iters = 1024
    e0.record(stream)
    cr.convrot_probe_i8_peak(iters, operands=operands, ws=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    iters = int(max(256, min(1 << 20, iters * burst_ms / max(e0.elapsed_time(e1), 1e-3))))
    ops = PROBE_OPS_PER_ITER_PER_PAIR * iters * pairs
    for _ in range(2):
        cr.convrot_probe_i8_peak(iters, operands=operands, ws=ws, stream=stream)
    torch.cuda.synchronize(dev)
    burst, burst_mhz = [], []
    with ClockSampler(clock_index, 0.001) as clk_b:
        for _ in range(10):
            e0.record(stream)
            cr.convrot_probe_i8_peak(iters, operands=operands, ws=ws, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            burst.append(ops / (e0.elapsed_time(e1) * 1e-3) / 1e12)
            burst_mhz.append(kernel_clock_mhz(ws))
    n_sus = int(max(1, sustained_s * 1e3 / burst_ms))
    with ClockSampler(clock_index, 0.005) as clk_s:
        e0.record(stream)
        for _ in range(n_sus):
            cr.convrot_probe_i8_peak(iters, operands=operands, ws=ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    sustained = ops * n_sus / (e0.elapsed_time(e1) * 1e-3) / 1e12
    sustained_mhz = kernel_clock_mhz(ws)  # the last launch of the loop
    if cr.convrot_read_device_status(ws) != 0:
        raise RuntimeError("int8 peak probe: a device wait timed out")
    b, s = clk_b.summary(), clk_s.summary()
    return {"peak_tops": max(max(burst), sustained),
            "burst_tops": max(burst), "burst_tops_median": statistics.median(burst), "sustained_tops": sustained,
            "burst_clock_mhz": b["sm_mhz"], "sustained_clock_mhz": s["sm_mhz"],
            "reasons": sorted(set(b["reasons"]) | set(s["reasons"])),
            "ops_per_clk_per_sm_burst": (max(burst) * 1e12 / (b["sm_mhz"] * 1e6) / ctas) if b["sm_mhz"] else None,
            "burst_sm_mhz_in_kernel": burst_mhz[burst.index(max(burst))],
            "sustained_sm_mhz_in_kernel": sustained_mhz,
            "ops_per_clk_per_sm_in_kernel": ((max(burst) * 1e12 / (burst_mhz[burst.index(max(burst))] * 1e6) / ctas)
                                             if burst_mhz[burst.index(max(burst))] else None),
            "probe": f"{pairs} CTA pairs x {iters} x 4 tcgen05.mma.cta_group::2.kind::i8 (256x256x32), "
                     f"zero operands in shared memory, no global traffic; burst = best of 10 launches of "
                     f"~{burst_ms:g} ms, sustained = {n_sus} launches back to back; peak = the larger of the two",
            "context": {"nominal_dense_int8_tops": NOMINAL_INT8_TOPS}}


def layer_inputs(cr, name: str, dev, up_cache: dict):
    """Device tensors of one config: X (bf16 [M,K]), the prepared weight, bias."""
    import synth
    import torch

    if name == "dit_mlp_down_1024":
        # the down projection's input is GELU of the up projection's output: the
        # up layer itself, with the GELU fused into its epilogue, produces it here
        if "down_x" not in up_cache:
            du = synth.make_workload("dit_mlp_up_1024")
            wq_u, sw_u = cr.convrot_prepare_weight(bits_to_dev(du["w"], dev), du["workload"].g)
            up_cache["down_x"] = cr.convrot_linear_ex(bits_to_dev(du["x"], dev), wq_u, sw_u, du["workload"].g, None,
                                                      cr.ACT_GELU_ERF)
            torch.cuda.synchronize(dev)
        w = synth.CONFIGS[name]
        rng = np.random.default_rng(w.seed)
        wt = rng.standard_normal((w.N, w.K), dtype=np.float32) * np.float32(w.w_std)
        Wq, sw = cr.convrot_prepare_weight(bits_to_dev(synth.f32_to_bf16_bits(wt), dev), w.g)
        return w, up_cache["down_x"], Wq, sw, None
    d = synth.make_workload(name)
    w = d["workload"]
    Wq, sw = cr.convrot_prepare_weight(bits_to_dev(d["w"], dev), w.g)
    bias = None if d["bias"] is None else bits_to_dev(d["bias"], dev)
    return w, bits_to_dev(d["x"], dev), Wq, sw, bias


def bench_config(cr, L, name: str, dev, stream, reps: int, peaks: dict, i8_peak, up_cache: dict) -> dict:
    """Per-config timing by CUDA events (median and min over `reps`), inputs rotated over buffer sets."""
    import torch

    w, X0, Wq0, sw, bias = layer_inputs(cr, name, dev, up_cache)
    M, K, N, g = w.M, w.K, w.N, w.g
    ws_bytes = cr.convrot_linear_workspace_bytes(M, N, K, g)
    per_set = 2.0 * M * K + N * K + 2.0 * M * N + ws_bytes
    ns = sets_for(per_set)
    sets = [{"X": X0 if i == 0 else X0.clone(), "Wq": Wq0 if i == 0 else Wq0.clone(),
             "Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
             "ws": torch.zeros((ws_bytes,), dtype=torch.uint8, device=dev),
             "Xq": torch.empty((M, K), dtype=torch.int8, device=dev),
             "sx": torch.empty((M,), dtype=torch.float32, device=dev)} for i in range(ns)]
    sp = stream.cuda_stream
    b_ptr = None if bias is None else bias.data_ptr()

    def call(i):
        s = sets[i % ns]
        st = L.convrot_linear(s["X"].data_ptr(), M, K, g, s["Wq"].data_ptr(), sw.data_ptr(), N, b_ptr,
                              s["Y"].data_ptr(), s["ws"].data_ptr(), ws_bytes, sp)
        if st != 0:
            raise cr.ConvRotError(st, f"convrot_linear ({name})")

    for i in range(5):
        call(i)
    torch.cuda.synchronize(dev)
    # back to back (the two launches of a call overlap as in a real forward pass)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(reps):
        call(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_b2b = e0.elapsed_time(e1) / reps
    # per call and per kernel: events before, between and after the two launches
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for trip in ev:
        for e in trip:
            e.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(reps):
        s = sets[i % ns]
        st = L.convrot_linear_timed(s["X"].data_ptr(), M, K, g, s["Wq"].data_ptr(), sw.data_ptr(), N, b_ptr,
                                    s["Y"].data_ptr(), s["ws"].data_ptr(), ws_bytes, ev[i][0].cuda_event,
                                    ev[i][1].cuda_event, ev[i][2].cuda_event, sp)
        if st != 0:
            raise cr.ConvRotError(st, f"convrot_linear_timed ({name})")
    torch.cuda.synchronize(dev)
    t_q_in = [e[0].elapsed_time(e[1]) for e in ev]
    t_g_in = [e[1].elapsed_time(e[2]) for e in ev]
    # the rotate+quantise pass alone, each launch between its own events
    evq = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for i in range(reps):
        s = sets[i % ns]
        evq[i][0].record(stream)
        L.convrot_quant_act(s["X"].data_ptr(), M, K, g, s["Xq"].data_ptr(), s["sx"].data_ptr(), sp)
        evq[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t_q = [e[0].elapsed_time(e[1]) for e in evq]
    for s in sets:
        if cr.convrot_read_device_status(s["ws"]) != 0:
            raise RuntimeError(f"{name}: device status not OK")
    ops = 2.0 * M * N * K
    q_bytes = 3.0 * M * K + 4.0 * M
    gq_med, gq_min = med_min(t_q)
    qi_med, qi_min = med_min(t_q_in)
    gg_med, gg_min = med_min(t_g_in)
    hbm = peaks["hbm_gbs"]
    out = {
        "M": M, "K": K, "N": N, "g": g, "sets": ns,
        "layer_us": t_b2b * 1e3, "layer_tops": ops / (t_b2b * 1e-3) / 1e12,
        "gemm_us_median": gg_med * 1e3, "gemm_us_min": gg_min * 1e3,
        "gemm_tops_median": ops / (gg_med * 1e-3) / 1e12,
        "quant_us_median": gq_med * 1e3, "quant_us_min": gq_min * 1e3,
        "quant_gbs_median": q_bytes / (gq_med * 1e-3) / 1e9, "quant_gbs_best": q_bytes / (gq_min * 1e-3) / 1e9,
        "quant_frac_hbm_median": q_bytes / (gq_med * 1e-3) / 1e9 / hbm,
        "quant_in_step_us_median": qi_med * 1e3,
        "quant_in_step_frac_hbm": q_bytes / (qi_med * 1e-3) / 1e9 / hbm,
    }
    if L.convrot_linear_launch_count(M, N, K, g) == 1:
        # one kernel rotates, quantises and multiplies: the "GEMM" events bracket all of it
        out["layer_kernels"] = "one (tokens quantised inside the weight-streaming GEMM)"
        out["quant_in_step_us_median"] = None
        out["quant_in_step_frac_hbm"] = None
    if i8_peak:
        out["gemm_frac_i8_peak_median"] = out["gemm_tops_median"] / i8_peak
    if M <= 128:
        # weight-streaming regime: bound by HBM on the algorithmic bytes of the layer
        gbytes = float(M * K + N * K + 2 * M * N + (2 * N if bias is not None else 0))
        out["layer_weight_stream_frac_hbm"] = gbytes / (t_b2b * 1e-3) / 1e9 / hbm
        out["gemm_weight_stream_frac_hbm"] = gbytes / (gg_med * 1e-3) / 1e9 / hbm
        out["algorithmic_bytes"] = gbytes
    del sets
    torch.cuda.empty_cache()
    return out


SFU_EX2_PER_CLK_PER_SM = 16  # special-function unit throughput of exp2 per SM per clock (B200)


def bench_attention(cr, dev, stream, reps: int, clock_index: int, i8_peak) -> dict:
    """INT8 attention at the pages' shape: 4096 image + 128 prefix tokens, 32 heads, head dim 128."""
    import torch

    BH, S, D = 32, 4224, 128
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    ns = 4  # 4 x (Q, K, V, O) = 553 MB: no call finds its inputs in L2
    sets = []
    for _ in range(ns):
        q, k, v = (torch.randn((BH, S, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(3))
        ws = torch.zeros((cr.convrot_attention_workspace_bytes(BH, S, S, D),), dtype=torch.uint8, device=dev)
        sets.append((q, k, v, torch.empty_like(q), ws))

    def call(i):
        q, k, v, o, ws = sets[i % ns]
        cr.convrot_attention_int8(q, k, v, O=o, ws=ws, stream=stream)

    for i in range(3):
        call(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(clock_index, 0.002) as clk:
        e0.record(stream)
        for i in range(reps):
            call(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    t_ms = e0.elapsed_time(e1) / reps
    for s in sets:
        if cr.convrot_read_device_status(s[4]) != 0:
            raise RuntimeError("attention: device status not OK")
    ops = 4.0 * S * S * D * BH  # Q K^T and P V
    exps = float(S) * S * BH
    c = clk.summary()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = c["sm_mhz"] or c["sm_max_mhz"] or 1965
    nominal = SFU_EX2_PER_CLK_PER_SM * sms * mhz * 1e6
    # the special-function unit's exp2 rate measured on this GPU (probe: independent ex2 chains)
    L = cr.lib()
    pws = torch.empty((256,), dtype=torch.float32, device=dev)
    per_iter = float(L.convrot_probe_ex2_per_iter())
    iters = 4096
    for _ in range(2):
        L.convrot_probe_ex2_peak(iters, pws.data_ptr(), pws.numel() * 4, stream.cuda_stream)
    e0.record(stream)
    for _ in range(5):
        L.convrot_probe_ex2_peak(iters, pws.data_ptr(), pws.numel() * 4, stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    measured = per_iter * iters * 5 / (e0.elapsed_time(e1) * 1e-3)
    out = {"BH": BH, "S": S, "D": D, "call_us": t_ms * 1e3, "tops": ops / (t_ms * 1e-3) / 1e12,
           "bound": "alu", "exp2_per_s": exps / (t_ms * 1e-3), "exp2_peak_per_s": measured,
           "frac_exp2_peak": exps / (t_ms * 1e-3) / measured, "clock_mhz": c["sm_mhz"],
           "exp2_peak_source": "measured: independent ex2.approx chains over a full grid (convrot_probe_ex2_peak)",
           "exp2_nominal_16_per_sm_clk": nominal,
           "note": "one call = rotate+quantise of Q and of K, the attention kernel"}
    if i8_peak:
        out["tensor_floor_us"] = (2.0 * S * S * D * BH / i8_peak + 2.0 * S * S * D * BH / (i8_peak / 2.0)) / 1e6
    del sets
    torch.cuda.empty_cache()
    return out


def e2e_overlapped(cr, d, X_sets, Wq_sets, sw, bias, g, Y_sets, ws_sets, dev, io_dtype, steps, warmup, barrier,
                   max_over_ranks, act=None, world=1):
    """The metric through the public API with host buffers: per step the input is
    copied from pinned host memory, the layer runs, and its output is copied back
    to pinned host memory, on three streams ordered by events over the buffer sets."""
    import torch

    ns = len(X_sets)
    M, K = X_sets[0].shape
    N = Wq_sets[0].shape[0]
    xh = [bits_to_dev(d["x"], "cpu", io_dtype).pin_memory() for _ in range(2)]
    yh = [torch.empty((M, N), dtype=io_dtype).pin_memory() for _ in range(2)]
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(ns)]
    ev_run = [torch.cuda.Event() for _ in range(ns)]
    ev_out = [torch.cuda.Event() for _ in range(ns)]
    used = [False] * ns

    def step(i):
        j = i % ns
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ev_run[j])  # the layer that last read X_j is done
            X_sets[j].copy_(xh[i % 2], non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[j])
            if used[j]:
                s_run.wait_event(ev_out[j])  # Y_j has been copied out
            if act is None:
                cr.convrot_linear(X_sets[j], Wq_sets[j], sw, g, bias, Y=Y_sets[j], ws=ws_sets[j], stream=s_run)
            else:
                cr.convrot_linear_ex(X_sets[j], Wq_sets[j], sw, g, bias, act, Y=Y_sets[j], ws=ws_sets[j],
                                     stream=s_run)
            ev_run[j].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[j])
            yh[i % 2].copy_(Y_sets[j], non_blocking=True)
            ev_out[j].record(s_out)
        used[j] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(dev)
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_run.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(steps):
        step(warmup + i)
    t1.record(s_out)
    s_out.synchronize()
    torch.cuda.synchronize(dev)
    barrier()
    t_ms = max_over_ranks(t0.elapsed_time(t1))
    ops = 2.0 * M * N * K
    return {"value": job_tops(ops, steps, world, t_ms), "unit": UNIT,
            "h2d_bytes_per_step": int(xh[0].numel() * xh[0].element_size()),
            "d2h_bytes_per_step": int(yh[0].numel() * yh[0].element_size()),
            "steps": steps, "ms_per_step": t_ms / steps,
            "schedule": f"host-to-device copy, layer and device-to-host copy on three streams, "
                        f"ordered by events over {ns} buffer sets"}


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import synth
    import w8a8_rotated_int8_token_b200 as cr

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the ConvRot path has no CPU implementation)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dev)

    if args.attention_only:
        att = bench_attention(cr, dev, torch.cuda.current_stream(dev), args.config_reps, local, None)
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"attention_int8_4224": att}), flush=True)
        return 0

    d = synth.make_workload(args.config)
    w = d["workload"]
    M, K, N, g = w.M, w.K, w.N, w.g
    L = cr.lib()

    variant = (args.dtype, args.wscale, args.act) != ("bf16", "tensor", "none")
    io_dtype = torch.bfloat16 if args.dtype == "bf16" else torch.float16
    dt_code = cr.DTYPE_BF16 if args.dtype == "bf16" else cr.DTYPE_F16
    ws_mode = cr.WSCALE_TENSOR if args.wscale == "tensor" else cr.WSCALE_CHANNEL
    act_code = cr.ACT_NONE if args.act == "none" else cr.ACT_GELU_ERF

    def to_dev(bits):
        return bits_to_dev(bits, dev, io_dtype)  # fp16: the same values rounded to fp16

    W = to_dev(d["w"])
    if variant:
        Wq0, sw = cr.convrot_prepare_weight_ex(W, g, ws_mode)
    else:
        Wq0, sw = cr.convrot_prepare_weight(W, g)
    del W
    bias = None if d["bias"] is None else to_dev(d["bias"])
    X0 = to_dev(d["x"])
    ws_bytes = cr.convrot_linear_workspace_bytes(M, N, K, g)
    sets = []
    for i in range(N_SETS):
        sets.append({
            "X": X0.clone(), "Wq": Wq0.clone(),
            "Y": torch.empty((M, N), dtype=io_dtype, device=dev),
            "ws": torch.zeros((ws_bytes,), dtype=torch.uint8, device=dev),
        })
    del X0
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    b_ptr = None if bias is None else bias.data_ptr()
    sw_ptr = sw.data_ptr()

    def step(i):
        s = sets[i % N_SETS]
        if variant:
            st = L.convrot_linear_ex(s["X"].data_ptr(), dt_code, M, K, 0, g, s["Wq"].data_ptr(), sw_ptr, ws_mode,
                                     N, b_ptr, None, act_code, s["Y"].data_ptr(), 0, s["ws"].data_ptr(), ws_bytes,
                                     sp)
        else:
            st = L.convrot_linear(s["X"].data_ptr(), M, K, g, s["Wq"].data_ptr(), sw_ptr, N, b_ptr,
                                  s["Y"].data_ptr(), s["ws"].data_ptr(), ws_bytes, sp)
        if st != 0:
            raise cr.ConvRotError(st, "convrot_linear")

    # ---- device-resident timed region
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    t_ms = max_over_ranks(ev0.elapsed_time(ev1))
    for s in sets:
        st = cr.convrot_read_device_status(s["ws"])
        if st != 0:
            raise cr.ConvRotError(st, "device status after the timed region")
    ops = 2.0 * M * N * K
    value = job_tops(ops, args.steps, world, t_ms)

    # ---- the layer kernel timed per launch: events recorded around each call on its stream
    launches = L.convrot_linear_launch_count(M, N, K, g)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for trip in ev:
        for e in trip:
            e.record(stream)  # creates the underlying cudaEvent_t
    torch.cuda.synchronize(dev)

    def timed_step(i, trip):
        s = sets[i % N_SETS]
        st = L.convrot_linear_timed(s["X"].data_ptr(), M, K, g, s["Wq"].data_ptr(), sw_ptr, N, b_ptr,
                                    s["Y"].data_ptr(), s["ws"].data_ptr(), ws_bytes, trip[0].cuda_event,
                                    trip[1].cuda_event, trip[2].cuda_event, sp)
        if st != 0:
            raise cr.ConvRotError(st, "convrot_linear_timed")

    if not variant:
        # Start this timed region from an idle GPU, as the probe's bursts do: right
        # after the headline loop the GPU still holds the lower clock its power limit
        # set there (the clock record below says which clock the GEMM ran at).
        time.sleep(IDLE_BEFORE_REGION_S)
        for i in range(max(args.warmup, WARMUP_AFTER_IDLE)):
            timed_step(i, ev[i % len(ev)])
        torch.cuda.synchronize(dev)
        barrier()
        for i in range(args.steps):
            timed_step(i, ev[i])
        torch.cuda.synchronize(dev)
        barrier()
        t_layer = max_over_ranks(statistics.mean(e[0].elapsed_time(e[2]) for e in ev))
        t_first = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev))
        t_first_med = max_over_ranks(statistics.median(e[0].elapsed_time(e[1]) for e in ev))
        t_second = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in ev))
        t_second_med = max_over_ranks(statistics.median(e[1].elapsed_time(e[2]) for e in ev))
        t_second_min = max_over_ranks(min(e[1].elapsed_time(e[2]) for e in ev))
        # the SM clock the GEMM ran at inside the steps: the clock record of each set's last call
        gemm_mhz = [m for m in (kernel_clock_mhz(s["ws"]) for s in sets) if m]
        gemm_mhz = statistics.median(gemm_mhz) if gemm_mhz else None
    else:
        gemm_mhz = None
    # (variants: no per-launch events; the GEMM's time is the layer's minus the
    # standalone rotate+quantise kernel's, below)

    # ---- the two stages as standalone kernels, each timed alone back to back (context)
    xq = [torch.empty((M, K), dtype=torch.int8, device=dev) for _ in range(N_SETS)]
    xsc = [torch.empty((M,), dtype=torch.float32, device=dev) for _ in range(N_SETS)]
    gws = torch.empty((L.convrot_gemm_workspace_bytes(),), dtype=torch.uint8, device=dev)

    def q_only(i):
        j = i % N_SETS
        if variant:
            L.convrot_quant_act_ex(sets[j]["X"].data_ptr(), dt_code, M, K, 0, g, xq[j].data_ptr(),
                                   xsc[j].data_ptr(), sp)
        else:
            L.convrot_quant_act(sets[j]["X"].data_ptr(), M, K, g, xq[j].data_ptr(), xsc[j].data_ptr(), sp)

    def g_only(i):
        j = i % N_SETS
        L.convrot_gemm_dequant(xq[j].data_ptr(), xsc[j].data_ptr(), sets[j]["Wq"].data_ptr(), sw_ptr, M, N, K,
                               b_ptr, sets[j]["Y"].data_ptr(), gws.data_ptr(), gws.numel(), sp)

    def time_loop(fn, n):
        for i in range(min(args.warmup, 10)):
            fn(i)
        torch.cuda.synchronize(dev)
        barrier()
        ev0.record(stream)
        for i in range(n):
            fn(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(ev0.elapsed_time(ev1)) / n

    n_alone = max(1, min(args.steps, 200))
    t_q = time_loop(q_only, n_alone)
    t_g = None if variant else time_loop(g_only, n_alone)
    if variant:
        t_layer = t_ms / args.steps
        t_first = t_q
        t_second = t_layer - t_q

    peaks, peak_src = load_peaks()
    # ---- the int8 tensor pipe's measured peak (the GEMM's roofline denominator)
    i8 = None
    if not args.no_peak:
        # the probe's operand tiles on the layer's own codes: 16 KB of activation codes
        # and 16 KB of weight codes per CTA
        n_ctas = int(L.convrot_probe_i8_peak_ctas())
        half = 16384
        codes = torch.stack([xq[0].view(-1)[: n_ctas * half].view(torch.uint8).view(n_ctas, half),
                             sets[0]["Wq"].view(-1)[: n_ctas * half].view(torch.uint8).view(n_ctas, half)],
                            1).contiguous() if M * K >= n_ctas * half and N * K >= n_ctas * half else None
        i8 = measure_i8_peak(cr, dev, stream, local, operands=codes)
        del codes
        i8["peak_tops"] = max_over_ranks(i8["peak_tops"])  # every rank runs it; the figure is per GPU
    del xq, xsc
    # The roofline denominator: the probe's rate on the layer's own codes (the data the
    # GEMM multiplies: the tensor cores draw more power on it than on zeros, and the GPU
    # holds a lower clock); the zero-operand rate is reported beside it.
    # A timed region of at most PEAK_BURST_REGION_MS is compared with the probe's burst
    # rate (single launches of ~5 ms), a longer one with its sustained rate (0.4 s back
    # to back), since the GPU lowers its clock under its power limit within tens of ms.
    int8_peak_zero = i8["peak_tops"] if i8 else None
    int8_peak_codes = None
    region_ms = t_ms
    peak_kind = "burst" if region_ms <= PEAK_BURST_REGION_MS else "sustained"
    int8_peak_short = int8_peak_zero  # for the configs' short repetitions: the burst rate on codes
    if i8 and "on_layer_codes" in i8:
        int8_peak_codes = max_over_ranks(i8["on_layer_codes"][f"{peak_kind}_tops"])
        int8_peak_short = max_over_ranks(i8["on_layer_codes"]["burst_tops"])
    if int8_peak_codes is not None:
        int8_peak = int8_peak_codes
        int8_peak_src = (f"measured int8 probe on the layer's own codes, {peak_kind} rate (the timed region lasted "
                         f"{region_ms:.1f} ms): tcgen05.mma.cta_group::2.kind::i8 from shared memory, operand tiles "
                         "copied from this layer's activation and weight codes")
    elif i8:
        int8_peak = int8_peak_zero
        int8_peak_src = ("measured int8 probe on zero operands (tcgen05.mma.cta_group::2.kind::i8 from shared memory; "
                         "the larger of its burst and sustained rates)")
    else:
        int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
        int8_peak_src = (f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {INT8_OVER_BF16} "
                         "(nominal int8:bf16 dense ratio)")
    layer_tops = ops / (t_layer * 1e-3) / 1e12
    gemm_tops = None if t_g is None else ops / (t_g * 1e-3) / 1e12
    q_bytes = 3.0 * M * K + 4.0 * M
    q_gbs = q_bytes / (t_q * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers (copies overlapped on streams)
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 100))
        e2e = e2e_overlapped(cr, d, [s["X"] for s in sets], [s["Wq"] for s in sets], sw, bias, g,
                             [s["Y"] for s in sets], [s["ws"] for s in sets], dev, io_dtype, e2e_steps,
                             min(args.warmup, 5), barrier, max_over_ranks,
                             act=(act_code if variant else None), world=world)
        if variant:
            e2e["note"] = "variant layer through convrot_linear_ex"

    cpu = None
    parity = None
    # the oracle leg reproduces the headline layer; variants report none
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not variant:
        y_all = sets[(args.steps - 1) % N_SETS]["Y"].float().cpu().numpy().astype(np.float64)
        cpu, parity = cpu_oracle_leg(d, args.cpu_seconds, y_all)
    del sets
    torch.cuda.empty_cache()

    # ---- every config of the workload table (device events; rank 0 prints)
    configs = None
    if not args.no_configs and not variant:
        configs = {}
        up_cache = {}
        shift = int(time.time() // 60) % len(CONFIG_NAMES)  # rotate the order from run to run
        order = CONFIG_NAMES[shift:] + CONFIG_NAMES[:shift]
        for name in order:
            configs[name] = bench_config(cr, L, name, dev, stream, args.config_reps, peaks,
                                         int8_peak_short if i8 else None, up_cache)
        configs["attention_int8_4224"] = bench_attention(cr, dev, stream, args.config_reps, local,
                                                         int8_peak_short if i8 else None)
        configs = {"order": order, "reps": args.config_reps,
                   "timing": "CUDA events on the launching stream; median and min over the repetitions; "
                             "layer_us from back-to-back calls",
                   "int8_peak_tops": int8_peak_short,
                   "int8_peak_source": "the int8 probe's burst rate on the default layer's codes", **configs}
        del up_cache

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    # the dominant kernel: the GEMM (second launch)
    t_dom = t_second
    dom_tops = ops / (t_dom * 1e-3) / 1e12
    hbm = peaks["hbm_gbs"]
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": workload_config(w),
        "pct_int8_peak": 100.0 * value / world / int8_peak,
        "roofline": {"bound": "tensor",
                     "kernel": "gemm_i8_pair_kernel (tcgen05.mma.cta_group::2 kind::i8, dequant/bias epilogue)",
                     "achieved": dom_tops, "peak": int8_peak, "unit": "TOPS", "frac": dom_tops / int8_peak,
                     "traffic": gemm_traffic(args.config) if not variant else None,
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "us_per_launch": t_dom * 1e3,
                     "us_source": ("layer time minus the standalone rotate+quantise kernel" if variant
                                   else "CUDA events around the GEMM launch inside each step (mean)"),
                     "peak_source": int8_peak_src,
                     "peak_zero_operands": int8_peak_zero,
                     "frac_zero_operands": (dom_tops / int8_peak_zero) if int8_peak_zero else None,
                     "peak_context": {"nominal_dense_int8_tops": NOMINAL_INT8_TOPS,
                                      "bf16_x2_tops": peaks["bf16_tflops"] * INT8_OVER_BF16,
                                      "bf16_source": peak_src}},
        "layer_us_per_call_events": t_layer * 1e3,
        "kernels": {
            "rotate_quant_kernel (first launch of the step, events)": ({
                "us": t_first * 1e3, "bound": "hbm", "achieved": q_bytes / (t_first * 1e-3) / 1e9, "unit": "GB/s",
                "peak": hbm, "frac": q_bytes / (t_first * 1e-3) / 1e9 / hbm,
                "us_median": (t_first_med * 1e3) if not variant else None} if launches == 2 else
                "none: one kernel rotates, quantises and multiplies (the tokens in shared memory)"),
            "rotate_quant_kernel (standalone, timed alone)": {
                "us": t_q * 1e3, "bound": "hbm", "achieved": q_gbs, "unit": "GB/s", "peak": hbm,
                "frac": q_gbs / hbm, "algorithmic_bytes": q_bytes},
        },
        "hbm_peak_source": f"{peak_src} copy bandwidth {hbm} GB/s",
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if not variant:
        out["roofline"]["us_per_launch_median"] = t_second_med * 1e3
        out["roofline"]["us_per_launch_min"] = t_second_min * 1e3
        out["roofline"]["sm_mhz_in_kernel"] = gemm_mhz
        opc = (i8 or {}).get("on_layer_codes", {}).get("ops_per_clk_per_sm_in_kernel")
        if gemm_mhz and opc and M > SMALL_M:
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            at_clock = opc * sms * gemm_mhz * 1e6 / 1e12
            out["roofline"]["peak_at_kernel_clock"] = at_clock
            out["roofline"]["frac_at_kernel_clock"] = dom_tops / at_clock
            out["roofline"]["clock_note"] = (
                "sm_mhz_in_kernel: the SM clock the GEMM ran at inside the steps (its %clock64 against "
                "%globaltimer); peak_at_kernel_clock: the probe's int8 rate per SM clock on the layer's codes "
                "times that clock; NVML's clock samples do not follow these changes")
    if i8:
        out["int8_peak"] = i8
    if M <= SMALL_M:
        # the weight-streaming GEMM (tokens as the MMA's N side): bound by HBM on the
        # weight bytes; algorithmic bytes M*K + N*K + 2*M*N (+ 2*N bias) per launch
        gbytes = float(M * K + N * K + 2 * M * N + (2 * N if bias is not None else 0))
        gbs = gbytes / (t_dom * 1e-3) / 1e9
        out["roofline"].update({
            "bound": "hbm", "kernel": "gemm_i8_smallm_kernel (swap-AB tcgen05 kind::i8, weight streaming" +
                                      (", tokens rotated and quantised in shared memory)" if launches == 1 else ")"),
            "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "algorithmic_bytes": gbytes, "traffic": None,
            "peak_source": f"{peak_src} HBM copy bandwidth {hbm} GB/s"})
    if variant:  # no per-launch events in a variant run: only the standalone timing is real
        del out["kernels"]["rotate_quant_kernel (first launch of the step, events)"]
    if t_g is not None:
        out["kernels"]["gemm_i8_kernel (GEMM + epilogue only, timed alone incl. 4-byte status memset)"] = {
            "us": t_g * 1e3, "bound": "tensor", "achieved": gemm_tops, "unit": "TOPS", "peak": int8_peak,
            "frac": gemm_tops / int8_peak, "ops": ops}
    if variant:
        out["config"]["variant"] = {"io_dtype": args.dtype, "weight_scale": args.wscale, "activation": args.act}
    if configs is not None:
        out["configs"] = configs
    if parity is not None:
        out["parity_nrmse_vs_oracle_sample"] = parity
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
