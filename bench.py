#!/usr/bin/env python
"""Benchmark of the W8A8 SmoothQuant linear path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode8b] [--impl ours]

One step = one pass of the whole hot path over one batch: for each token count M of the
workload, one Llama decoder block's linear path on its own layer's weights
(smoothed RMSNorm+quant -> qkv GEMM; attention stand-in -> quant -> o GEMM; residual add ->
smoothed RMSNorm+quant -> gate_up GEMM; SiLU*up+quant -> down GEMM). The default workload is
the Llama-3.1-8B decode set, M = 1, 8, 32, 64 (four layers, 872 MB of int8 weights, so
every step streams its weights from HBM: inputs larger than L2, no flush needed).

The timed region replays a CUDA graph of the step K times between CUDA events on the
launching stream, after W warm-up steps, bracketed by a barrier and device synchronizations;
multi-GPU runs are independent replicas (one process per GPU, no data-path collective) and
report the max time over ranks. Prints one JSON line (rank 0).

`--impl reference` times the CPU oracle instead (host cores, bounded samples of the same
workload). `--case gemm:M:N:K` runs one GEMM launch repeatedly (for profilers).
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "W8A8 linear TOPS & HBM GB/s at Llama-3.1-8B shapes; % of roofline"
EPS = 1e-5
ALPHA = 0.5
CALIB_TOKENS = 128

LLAMA8B = dict(model="llama-3.1-8b", H=4096, I=14336, QKV=6144)
LLAMA70B = dict(model="llama-3.1-70b", H=8192, I=28672, QKV=10240)
WORKLOADS = {
    "decode8b": dict(arch=LLAMA8B, Ms=[1, 8, 32, 64], desc="Llama-3.1-8B decode linear set"),
    "prefill8b": dict(arch=LLAMA8B, Ms=[2048, 8192], desc="Llama-3.1-8B prefill linear set"),
    "block8b": dict(arch=LLAMA8B, Ms=[512], desc="Llama-3.1-8B decoder block linear path"),
    "set70b": dict(arch=LLAMA70B, Ms=[16, 4096], desc="Llama-3.1-70B-shaped linear set"),
}

# DRAM bytes (read + write, ncu dram__bytes_read.sum + dram__bytes_write.sum) per GEMM launch,
# averaged over the GEMM launches of one step of the workload, as captured with the current
# GEMM kernels; None where no capture exists. Re-capture whenever a GEMM kernel changes.
NCU_GEMM_TRAFFIC = {"decode8b": 54.86e6, "prefill8b": 226.2e6}

# Measured peaks (driver-written); fallbacks are the pool's earlier measurements.
FALLBACK_HBM_GBS = 6650.0
INT8_NOMINAL_TOPS = 4500.0


# ------------------------------------------------------------------ work model


def projections(arch):
    H, I, Q = arch["H"], arch["I"], arch["QKV"]
    return {"qkv": (Q, H), "o": (H, H), "gate_up": (2 * I, H), "down": (H, I)}


def gemm_bytes(M, N, K):
    """Algorithmic HBM bytes of one GEMM+dequant: int8 weight and activation, fp32 scales,
    bf16 output."""
    return N * K + M * K + 4 * M + 4 * N + 2 * M * N


def layer_work(arch, M):
    """(ops, bytes, gemm_ops, gemm_bytes) of one block's linear path at M tokens."""
    H, I = arch["H"], arch["I"]
    P = projections(arch)
    g_ops = sum(2 * M * N * K for (N, K) in P.values())
    g_bytes = sum(gemm_bytes(M, N, K) for (N, K) in P.values())
    row_bytes = ((3 * M * H + 4 * M + 4 * H)          # smoothed RMSNorm + quant (qkv input)
                 + (3 * M * H + 4 * M + 4 * H)        # quantize_rows (o input, smoothed)
                 + (7 * M * H + 4 * M + 4 * H)        # residual add + RMSNorm + quant
                 + (5 * M * I + 4 * M))               # SiLU*up + quant (down input)
    return g_ops, g_bytes + row_bytes, g_ops, g_bytes


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ distributed plumbing


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def reduce_max(value: float) -> float:
    """Max of a float over ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def combine(units_per_rank: float, seconds_per_rank: float, world: int):
    """Whole-job throughput of `world` replicas: all units over the slowest rank's time."""
    t = reduce_max(seconds_per_rank)
    return units_per_rank * world / t, t


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) in a thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting"}

    def __init__(self, device_index, period_s=0.05):
        self.samples = []
        self.err = None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report why
            self.err = repr(e)
            self.h = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception as e:
                self.err = repr(e)
            time.sleep(self.period)

    def start(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.h is not None:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if self.h is None:
            return {"error": self.err}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "during the timed region"
        if len(win) < 3:
            win = [s for s in self.samples if s[0] >= t0]
            note = "timed region plus the same load replayed right after it"
        if not win:
            return {"error": "no samples", "sm_max_mhz": self.max_mhz}
        reasons = set()
        for _, _, rs in win:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win), "window": note}


# ------------------------------------------------------------------ workload on the GPU


class Layer:
    """One decoder block's linear path at M tokens: prepared weights, inputs, outputs."""

    def __init__(self, arch, M, seed, device, fp8=False, block=False):
        import int8_w8a8_quantized_smoothed_b200 as w8
        from int8_w8a8_quantized_smoothed_b200 import prep, synth
        self.M, self.arch, self.fp8 = M, arch, fp8
        H, I = arch["H"], arch["I"]
        P = projections(arch)
        g1 = synth.gamma_device(H, seed + 1, device)
        g2 = synth.gamma_device(H, seed + 2, device)
        # calibration batches (separate seeds, same distributions as the served tokens)
        x_cal = synth.activation_device(CALIB_TOKENS, H, seed + 3, device)
        a_cal = synth.activation_device(CALIB_TOKENS, H, seed + 4, device)
        h_cal = synth.activation_device(CALIB_TOKENS, H, seed + 5, device)
        a_qkv = prep.column_absmax(prep.rmsnorm_calibration(x_cal, g1, EPS))
        a_o = prep.column_absmax(a_cal)
        a_gu = prep.column_absmax(prep.rmsnorm_calibration(h_cal, g2, EPS))
        self.w = {}
        self.fused = True
        self.o_norm = True  # o GEMM + residual RMSNorm + quant through one entry point (INT8)
        self.o_norm_one_launch = False  # ... as the GEMM's row tail (decode sizes)
        for i, (name, (N, K)) in enumerate(P.items()):
            wb = synth.weight_device(N, K, seed + 10 + i, device)
            if name == "qkv":
                p = prep.prepare_linear(wb, a_qkv, ALPHA)
                self.g1f = torch.from_numpy(prep.fold(g1.cpu().numpy(), p["s"])[0]).to(device)
            elif name == "o":
                p = prep.prepare_linear(wb, a_o, ALPHA)
                self.sinv_o = p["s_inv_dev"]
            elif name == "gate_up":
                p = prep.prepare_linear(wb, a_gu, ALPHA)
                self.g2f = torch.from_numpy(prep.fold(g2.cpu().numpy(), p["s"])[0]).to(device)
            else:  # down: its input is SiLU*up, no norm to fold into
                wq, sch = w8.w8a8_quantize_rows(wb)
                p = dict(wq=wq, s_ch=sch, s_dev=None)
            if fp8:  # E4M3 codes of the same smoothed weight, scales absmax / 448
                self.w[name] = w8.w8a8_quantize_rows_fp8(wb, p["s_dev"])
            else:
                self.w[name] = (p["wq"], p["s_ch"])
            del wb, p
        # the gate|up weight in the row order of the fused SiLU*up epilogue
        self.w_gu_il = prep.interleave_gate_up(*self.w["gate_up"])
        torch.cuda.synchronize()
        # inputs (device) and their pinned host copies for the end-to-end measurement
        self.x = synth.activation_device(M, H, seed + 20, device)
        self.attn = synth.activation_device(M, H, seed + 21, device)
        self.x_host = self.x.cpu().pin_memory()
        self.attn_host = self.attn.cpu().pin_memory()
        e = dict(device=device)
        qt = w8.FP8 if fp8 else torch.int8
        self.q1 = torch.empty(M, H, dtype=qt, **e)
        self.s1 = torch.empty(M, dtype=torch.float32, **e)
        self.qkv = torch.empty(M, P["qkv"][0], dtype=torch.bfloat16, **e)
        self.q2 = torch.empty(M, H, dtype=qt, **e)
        self.s2 = torch.empty(M, dtype=torch.float32, **e)
        self.o = torch.empty(M, H, dtype=torch.bfloat16, **e)
        self.h = torch.empty(M, H, dtype=torch.bfloat16, **e)
        self.q3 = torch.empty(M, H, dtype=qt, **e)
        self.s3 = torch.empty(M, dtype=torch.float32, **e)
        self.gu = torch.empty(M, 2 * I, dtype=torch.bfloat16, **e)
        self.a = torch.empty(M, I, dtype=torch.float32, **e)  # SiLU*up of the fused path
        self.q4 = torch.empty(M, I, dtype=qt, **e)
        self.s4 = torch.empty(M, dtype=torch.float32, **e)
        self.down = torch.empty(M, H, dtype=torch.bfloat16, **e)
        self.down_host = torch.empty(M, H, dtype=torch.bfloat16).pin_memory()
        # the fused decoder-block kernel: its own buffers; the block output is self.down
        self.block = None
        if block:
            self.block = w8.BlockBuffers(M, H, I, P["qkv"][0], device)
            self.down = self.block.y

    def rows(self):
        import int8_w8a8_quantized_smoothed_b200 as w8
        w8.w8a8_smooth_rmsnorm_quant(self.x, self.g1f, EPS, q=self.q1, s_tok=self.s1)
        w8.w8a8_quantize_rows(self.attn, self.sinv_o, q=self.q2, s_tok=self.s2)

    def chain(self, ws, gemms=True, rows=True, fused=None):
        import int8_w8a8_quantized_smoothed_b200 as w8
        fused = self.fused if fused is None else fused
        if self.fp8:
            return self.chain_fp8(ws, gemms, rows, fused)
        if self.block is not None:  # one launch for the whole block
            w8.w8a8_block_decode(self.x, self.attn, self.g1f, self.sinv_o, self.g2f,
                                 self.w["qkv"], self.w["o"], self.w_gu_il, self.w["down"], EPS,
                                 buffers=self.block)
            return
        if rows:
            w8.w8a8_smooth_rmsnorm_quant(self.x, self.g1f, EPS, q=self.q1, s_tok=self.s1)
        if gemms:
            w8.w8a8_gemm_dequant(self.q1, self.s1, *self.w["qkv"], y=self.qkv, workspace=ws)
        if rows:
            w8.w8a8_quantize_rows(self.attn, self.sinv_o, q=self.q2, s_tok=self.s2)
        if gemms and rows and self.o_norm:
            # o projection, residual add and the next RMSNorm + quant: one call
            w8.w8a8_gemm_rmsnorm_quant(self.q2, self.s2, *self.w["o"], self.x, self.g2f, EPS,
                                       y=self.o, h_out=self.h, q=self.q3, s_out=self.s3,
                                       workspace=ws, one_launch=self.o_norm_one_launch)
        else:
            if gemms:
                w8.w8a8_gemm_dequant(self.q2, self.s2, *self.w["o"], y=self.o, workspace=ws)
            if rows:
                w8.w8a8_smooth_rmsnorm_quant(self.o, self.g2f, EPS, residual=self.x,
                                             h_out=self.h, q=self.q3, s_tok=self.s3)
        if fused:
            # gate|up GEMM with the SiLU*up epilogue, then its per-token quantization pass
            if gemms:
                w8.w8a8_gemm_silu_quant(self.q3, self.s3, *self.w_gu_il, a=self.a, q=self.q4,
                                        s_out=self.s4, workspace=ws)
        else:
            if gemms:
                w8.w8a8_gemm_dequant(self.q3, self.s3, *self.w["gate_up"], y=self.gu,
                                     workspace=ws)
            if rows:
                w8.w8a8_silu_mul_quant(self.gu, q=self.q4, s_tok=self.s4)
        if gemms:
            w8.w8a8_gemm_dequant(self.q4, self.s4, *self.w["down"], y=self.down, workspace=ws)


    def chain_fp8(self, ws, gemms=True, rows=True, fused=True):
        """The same block with E4M3 codes: FP8 row kernels and FP8 GEMMs."""
        import int8_w8a8_quantized_smoothed_b200 as w8
        if rows:
            w8.w8a8_smooth_rmsnorm_quant_fp8(self.x, self.g1f, EPS, q=self.q1, s_tok=self.s1)
        if gemms:
            w8.w8a8_gemm_dequant_fp8(self.q1, self.s1, *self.w["qkv"], y=self.qkv, workspace=ws)
        if rows:
            w8.w8a8_quantize_rows_fp8(self.attn, self.sinv_o, q=self.q2, s_tok=self.s2)
        if gemms:
            w8.w8a8_gemm_dequant_fp8(self.q2, self.s2, *self.w["o"], y=self.o, workspace=ws)
        if rows:
            w8.w8a8_smooth_rmsnorm_quant_fp8(self.o, self.g2f, EPS, residual=self.x,
                                             h_out=self.h, q=self.q3, s_tok=self.s3)
        if fused:
            if gemms:
                w8.w8a8_gemm_silu_quant_fp8(self.q3, self.s3, *self.w_gu_il, a=self.a,
                                            q=self.q4, s_out=self.s4, workspace=ws)
        else:
            if gemms:
                w8.w8a8_gemm_dequant_fp8(self.q3, self.s3, *self.w["gate_up"], y=self.gu,
                                         workspace=ws)
            if rows:
                w8.w8a8_silu_mul_quant_fp8(self.gu, q=self.q4, s_tok=self.s4)
        if gemms:
            w8.w8a8_gemm_dequant_fp8(self.q4, self.s4, *self.w["down"], y=self.down,
                                     workspace=ws)


def measure_int8_peak(iters=20000, reps=3, sustained_s=0.0):
    """Dense INT8 tensor-core rate of this device in TOPS from the library's tcgen05 kind::i8
    probe (128 x 256 x 32 MMAs back to back on every SM): the best of `reps` launches
    (burst), or with sustained_s > 0 the average over launches back to back for that many
    seconds (the rate under the power cap, for kernels timed inside a long step)."""
    import int8_w8a8_quantized_smoothed_b200 as w8
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    ops = 2 * 128 * 256 * 32 * iters * sms
    w8.w8a8_probe_i8_mma(1000)
    torch.cuda.synchronize()
    if sustained_s > 0:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n, t0 = 0, time.perf_counter()
        e0.record()
        while time.perf_counter() - t0 < sustained_s:
            for _ in range(10):
                w8.w8a8_probe_i8_mma(iters)
            n += 10
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
        return ops * n / (e0.elapsed_time(e1) / 1e3) / 1e12
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        w8.w8a8_probe_i8_mma(iters)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, ops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    return best


def capture(fn):
    """CUDA graph of fn() (warmed up on a side stream first)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, steps, warmup):
    """Seconds for `steps` replays (events on the launching stream), after `warmup`."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1) / 1e3


def replay_latencies(g, n):
    """Per-replay device times (microseconds) of n back-to-back replays: an event pair
    around every replay on the launching stream (the replays still follow one another
    without host synchronization). Returns p50, p95 and mean."""
    st = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    ev[0].record(st)
    for i in range(n):
        g.replay()
        ev[i + 1].record(st)
    torch.cuda.synchronize()
    t = sorted(ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(n))
    return {"p50_us": round(statistics.median(t), 2),
            "p95_us": round(t[min(n - 1, math.ceil(0.95 * n) - 1)], 2),
            "mean_us": round(sum(t) / n, 2), "n": n,
            "how": "one CUDA event pair per graph replay, replays back to back"}


def run_ours(args, world, rank, local):
    """The workload's JSON line; with the default decode workload it also carries a record
    of each --extra workload (prefill8b by default), measured the same way in this run."""
    import int8_w8a8_quantized_smoothed_b200 as w8
    from int8_w8a8_quantized_smoothed_b200 import build as wbuild
    wbuild.build()
    w8.lib()
    result = measure_workload(args, args.workload, world, rank, local, primary=True)
    extras = [] if args.extra in ("", "none") else [
        e for e in args.extra.split(",") if e != args.workload]
    for name in extras:
        torch.cuda.empty_cache()
        result[name] = measure_workload(args, name, world, rank, local, primary=False)
    return result


def measure_workload(args, name, world, rank, local, primary):
    """Times one workload's step (and its GEMM launches and row launches alone). The primary
    workload's record is the JSON line itself (with e2e and the CPU baseline); a secondary
    one is a nested record with the same timing, roofline and clock keys."""
    import int8_w8a8_quantized_smoothed_b200 as w8
    dev = torch.device("cuda", local)
    wl = WORKLOADS[name]
    arch = wl["arch"]
    layers = [Layer(arch, M, seed=1000 * (i + 1), device=dev, fp8=args.fp8,
                    block=args.fused_block) for i, M in enumerate(wl["Ms"])]
    unfused = args.unfused
    for L in layers:
        L.fused = not unfused
        L.o_norm_one_launch = args.o_norm_one_launch and L.M <= 64
    ws = w8.Workspace(dev)
    max_ws = max([w8.w8a8_gemm_workspace_size(L.M, N, K) for L in layers
                  for (N, K) in projections(arch).values()] +
                 [w8.w8a8_gemm_fp8_workspace_size(L.M, N, K) for L in layers
                  for (N, K) in projections(arch).values()] +
                 [w8.w8a8_gemm_silu_quant_workspace_size(L.M, arch["I"], arch["H"])
                  for L in layers] +
                 [w8.w8a8_gemm_rmsnorm_quant_workspace_size(L.M, arch["H"], arch["H"])
                  for L in layers] +
                 [w8.w8a8_gemm_silu_quant_fp8_workspace_size(L.M, arch["I"], arch["H"])
                  for L in layers])
    ws.get(max_ws)
    # the weights are prepared and synchronized: from here on no kernel writes them, so the
    # GEMMs may stream them ahead of the dependency wait (overlap mode 2)
    torch.cuda.synchronize()
    w8.w8a8_set_overlap(args.overlap)

    def step():
        for L in layers:
            L.chain(ws)

    def step_gemms():  # the GEMM kernels alone, plain dequant epilogues
        for L in layers:
            L.chain(ws, rows=False, fused=False)

    def step_gemms_fused():  # the step's GEMM-type launches incl. the SiLU*up quant pass
        for L in layers:
            L.chain(ws, rows=False)

    def step_rows():
        for L in layers:
            L.chain(ws, gemms=False)

    copy_stream = torch.cuda.Stream(device=dev)

    def step_e2e():
        # every input crosses to the device and every output back inside the step; the
        # copies run on their own stream, each layer waiting only for its own inputs and its
        # output leaving while the next layer computes
        main = torch.cuda.current_stream()
        copy_stream.wait_stream(main)
        ready = []
        with torch.cuda.stream(copy_stream):
            for L in layers:
                L.x.copy_(L.x_host, non_blocking=True)
                L.attn.copy_(L.attn_host, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
                ready.append(ev)
        for L, ev in zip(layers, ready):
            main.wait_event(ev)
            L.chain(ws)
            done = torch.cuda.Event()
            done.record(main)
            copy_stream.wait_event(done)
            with torch.cuda.stream(copy_stream):
                L.down_host.copy_(L.down, non_blocking=True)
        main.wait_stream(copy_stream)

    ops = sum(layer_work(arch, L.M)[0] for L in layers)
    nbytes = sum(layer_work(arch, L.M)[1] for L in layers)
    g_bytes = sum(layer_work(arch, L.M)[3] for L in layers)

    if args.fused_block:
        launches_per_step = len(layers)
    else:  # 8 per layer, 7 where the o GEMM runs the RMSNorm tail in the same launch
        launches_per_step = sum(8 - (1 if L.o_norm_one_launch and not args.fp8 else 0)
                                for L in layers)
    h2d = sum(L.x.numel() * 2 + L.attn.numel() * 2 for L in layers)
    d2h = sum(L.down.numel() * 2 for L in layers)

    int8_peak = measure_int8_peak()
    g_step = capture(step)
    assert w8.w8a8_device_status(reset=True) == 0, "device-side wait ran out"

    clocks = ClockSampler(local).start()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    secs = time_graph(g_step, args.steps, args.warmup)
    t_wall1 = time.perf_counter()
    # keep the same load running briefly if the timed region was too short to sample
    if t_wall1 - t_wall0 < 0.3 and clocks.h is not None:
        t_end = time.perf_counter() + 0.5
        while time.perf_counter() < t_end:
            for _ in range(50):
                g_step.replay()
            torch.cuda.synchronize()
    clocks.stop()
    value, t_max = combine(nbytes, secs / args.steps, world)
    ms_per_step = t_max * 1e3

    # dominant kernel: the GEMM launches of the step, timed alone as a graph (the fused block
    # kernel has no separate GEMM launches: its whole step stands in)
    if args.fused_block:
        g_gemm = g_rows = None
        gsecs, rsecs = t_max, 0.0
    else:
        g_gemm = capture(step_gemms)
        gsecs = time_graph(g_gemm, args.steps, args.warmup) / args.steps
        g_rows = capture(step_rows)
        rsecs = time_graph(g_rows, args.steps, args.warmup) / args.steps
    gfsecs = None
    if not unfused and not args.fused_block:
        g_gemm_f = capture(step_gemms_fused)
        gfsecs = time_graph(g_gemm_f, args.steps, args.warmup) / args.steps
        del g_gemm_f
    latency = replay_latencies(g_step, max(100, min(args.steps, 1000)))
    g_e2e = esecs = e_value = None
    if primary:
        g_e2e = capture(step_e2e)
        esecs = time_graph(g_e2e, args.steps, args.warmup) / args.steps
        e_value, _ = combine(nbytes, esecs, world)
    assert w8.w8a8_device_status(reset=True) == 0, "device-side wait ran out"

    hbm_peak, peak_src = read_peaks()
    gemm_gbs = g_bytes / gsecs / 1e9
    gemm_tops = ops / gsecs / 1e12
    t_roof = max(ops / (INT8_NOMINAL_TOPS * 1e12), nbytes / (hbm_peak * 1e9))
    t_roof_meas = max(ops / (int8_peak * 1e12), nbytes / (hbm_peak * 1e9))
    tensor_bound = ops / (int8_peak * 1e12) > g_bytes / (hbm_peak * 1e9)
    if tensor_bound:
        # the GEMMs run inside a long step under the power cap: the sustained probe rate is
        # the denominator; the burst rate and the nominal figure are reported beside it
        int8_sus = measure_int8_peak(sustained_s=3.0)
        roofline = {"kernel": "gemm_prefill_pair_kernel / gemm_prefill_kernel "
                              "(all GEMM launches of the step)",
                    "bound": "tensor", "achieved": round(gemm_tops, 1),
                    "peak": round(int8_sus, 1), "unit": "TFLOP/s",
                    "frac": round(gemm_tops / int8_sus, 4),
                    "peak_source": "measured: tcgen05 kind::i8 probe in this run, 3 s back to "
                                   "back (sustained)",
                    "peak_burst": round(int8_peak, 1),
                    "frac_of_burst": round(gemm_tops / int8_peak, 4),
                    "frac_of_nominal": round(gemm_tops / INT8_NOMINAL_TOPS, 4),
                    "traffic": None}
    else:
        roofline = {"kernel": ("block_decode_kernel (the fused block: the whole step, row "
                               "phases included)") if args.fused_block else
                              ("gemm_decode_kernel" + ("<F8>" if args.fp8 else "") +
                               " (all GEMM launches of the step, plain dequant epilogues, timed "
                               "alone as a graph)"),
                    "bound": "hbm", "achieved": round(gemm_gbs, 1), "peak": hbm_peak,
                    "unit": "GB/s", "frac": round(gemm_gbs / hbm_peak, 4),
                    "peak_source": f"{peak_src} copy bandwidth (burst)", "traffic": None}
    roofline["per_launch_us"] = round(gsecs / ((1 if args.fused_block else 4) * len(layers)) * 1e6, 3)
    result = {
        "metric": METRIC, "value": round(value / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("e4m3xe4m3->f32, fp32 scales, bf16 io" if args.fp8 else
                  "i8xi8->i32, fp32 scales, bf16 io"), "data": "synthetic",
        "config": {**workload_config(wl, arch), "parallelism": f"replicas x{world}",
                   "l2": "no flush: each step streams "
                         f"{sum(L.w[n][0].numel() for L in layers for n in L.w) / 1e6:.0f} MB "
                         "of int8 weights (> 126 MB L2)",
                   "timing": "CUDA graph of one step replayed K times, CUDA events",
                   "overlap": args.overlap,
                   "silu_mul_quant": ("separate launch" if unfused else
                                      "fused into the gate|up GEMM epilogue + quantization pass"),
                   "o_norm": ("residual add + RMSNorm + quant in the o GEMM's row tail "
                              "(M <= 64)" if args.o_norm_one_launch and not args.fp8 else
                              "separate launch (the faster form)"),
                   "codes": "FP8 E4M3 (scale absmax / 448)" if args.fp8 else
                            "INT8 (scale absmax / 127)"},
        "tops": round(ops / t_max / 1e12, 3),
        "latency_us": latency,
        "roofline_step": {"t_roof_us": round(t_roof * 1e6, 2),
                          "t_us": round(t_max * 1e6, 2), "frac": round(t_roof / t_max, 4),
                          "frac_vs_measured_int8": round(t_roof_meas / t_max, 4),
                          "note": "max(ops / 4.5 POPS nominal INT8, bytes / measured HBM)"},
        "int8_peak_tops_measured": round(int8_peak, 1),
        "roofline": roofline,
        "breakdown_us": {"step": round(t_max * 1e6, 2), "gemms": round(gsecs * 1e6, 2),
                         "row_kernels": round(rsecs * 1e6, 2),
                         **({"gemms_with_fused_silu_and_quant_pass": round(gfsecs * 1e6, 2)}
                            if gfsecs is not None else {}),
                         "note": "gemms: plain epilogues; row_kernels: the step's row "
                                 "launches" + ("" if unfused else
                                               " (SiLU*up is fused into the gate|up GEMM)")},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(t_wall0, time.perf_counter()),
    }
    if primary:
        result["e2e"] = {"value": round(e_value / 1e9, 2), "unit": "GB/s",
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                         "ms_per_step": round(esecs * 1e3, 5),
                         "how": "CUDA graph per step: pinned-host inputs H2D and outputs D2H on "
                                "a copy stream overlapping the other layers' C-ABI calls"}
    else:  # a nested record: the JSON line's own keys stay the primary workload's
        for k in ("metric", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                  "vs_baseline", "data", "gpu_launches"):
            result.pop(k)
    if primary and rank == 0 and world == 1 and not args.no_cpu_baseline and not args.fp8:
        result["cpu_baseline"] = cpu_baseline(arch)
    traffic = args.traffic if (args.traffic is not None and primary) else (
        None if args.fp8 else NCU_GEMM_TRAFFIC.get(name))
    if traffic is not None:
        result["roofline"]["traffic"] = traffic
        result["roofline"]["traffic_per"] = "GEMM launch (ncu DRAM read + write bytes)"
        result["roofline"]["algorithmic_bytes_per_launch"] = round(g_bytes / (4 * len(layers)))
    del g_step, g_gemm, g_rows, g_e2e, layers
    return result


# ------------------------------------------------------------------ oracle (CPU) legs


def _oracle_layer(arch, M, seed):
    """Inputs and prepared int8 weights for the oracle's chain (CPU, seeded)."""
    from int8_w8a8_quantized_smoothed_b200 import synth
    H = arch["H"]
    P = projections(arch)
    pr = {}
    for i, (name, (N, K)) in enumerate(P.items()):
        pr[name] = dict(wq=synth.int8_codes((N, K), seed + i, extremes=False),
                        s_ch=synth.scales(N, seed + 10 + i, 1e-4, 2e-2))
    pr["gamma1f"] = synth.gamma(H, seed + 20)
    pr["gamma2f"] = synth.gamma(H, seed + 21)
    pr["s_inv_o"] = (1.0 / synth.gamma(H, seed + 22)).astype(np.float32)
    inputs = dict(x=synth.activation(M, H, seed + 30), attn=synth.activation(M, H, seed + 31))
    return pr, inputs


def cpu_baseline(arch, M=64, min_seconds=10.0):
    """The oracle, as it stands, on this host's cores: one decoder block's linear path at
    M tokens, repeated for at least `min_seconds`."""
    import oracle
    pr, inputs = _oracle_layer(arch, M, 77)
    nthreads = oracle.NTHREADS
    _, nbytes, _, _ = layer_work(arch, M)
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.block_reference(inputs, pr, EPS, nthreads=nthreads)
        passes += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": round(nbytes * passes / el / 1e9, 4), "unit": "GB/s",
            "cores": min(nthreads, M), "kind": "oracle",
            "sample": f"one decoder block's linear path at M={M} ({arch['model']} shapes), "
                      f"{passes} passes in {el:.1f} s; rows split over {min(nthreads, M)} "
                      f"threads of {os.cpu_count()} host cores"}


def workload_config(wl, arch):
    """The workload's description, the same in both arms' JSON lines."""
    return {"workload": f"{wl['desc']}, M in {wl['Ms']}: one decoder block's linear path per M "
                        f"on its own layer's weights",
            "tokens": wl["Ms"], "hidden": arch["H"], "intermediate": arch["I"],
            "qkv_out": arch["QKV"], "alpha": ALPHA}


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle timed on the host cores, each step a bounded sample
    (the M=1 block linear path of the workload's architecture)."""
    if rank != 0:
        return None
    import oracle
    wl = WORKLOADS[args.workload]
    arch = wl["arch"]
    M = 1
    pr, inputs = _oracle_layer(arch, M, 91)
    _, nbytes, _, _ = layer_work(arch, M)
    nth = oracle.NTHREADS
    for _ in range(args.warmup):
        oracle.block_reference(inputs, pr, EPS, nthreads=nth)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.block_reference(inputs, pr, EPS, nthreads=nth)
    el = time.perf_counter() - t0
    value = nbytes * args.steps / el / 1e9
    sample = (f"per step: one decoder block's linear path at M={M} ({arch['model']} shapes) "
              f"through the CPU oracle")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8xi8->i32, fp32 scales, bf16 io",
        "data": "synthetic",
        "config": {**workload_config(wl, arch), "parallelism": "host cores",
                   "codes": "INT8 (scale absmax / 127)",
                   "sample": f"each step: the M={M} member of the set through the CPU oracle"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": min(nth, M),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ single-kernel case


def measure_f64_peak(iters=4000, reps=3):
    """Binary64 FMA rate (TFLOP/s) of this device from w8a8_probe_f64_fma, best of reps."""
    import int8_w8a8_quantized_smoothed_b200 as w8
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    ctas = props.multi_processor_count * 8
    out = torch.empty(ctas * 256, dtype=torch.float64, device="cuda")
    w8.w8a8_probe_f64_fma(iters, ctas, out)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        w8.w8a8_probe_f64_fma(iters, ctas, out)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, 2 * 8 * iters * 256 * ctas / (e0.elapsed_time(e1) / 1e3) / 1e12)
    return best


def run_gptq_case(args, dims):
    """`--case gptq:N:K:T`: GPTQ of one [N, K] weight with T calibration tokens, whole call
    (Hessian, factor, quantize-and-compensate) timed with CUDA events; binary64 flops against
    the FMA probe's rate."""
    import int8_w8a8_quantized_smoothed_b200 as w8
    from int8_w8a8_quantized_smoothed_b200 import build as wbuild, synth
    wbuild.build()
    N, K, T = dims
    dev = torch.device("cuda", 0)
    w = synth.weight_device(N, K, 1, dev)
    x = synth.activation_device(T, K, 2, dev).float()
    s = synth.gamma_device(K, 3, dev).float()
    ws = torch.empty(w8.w8a8_gptq_workspace_size(N, K), dtype=torch.uint8, device=dev)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    sch = torch.empty(N, dtype=torch.float32, device=dev)
    w8.w8a8_gptq_quantize(w, x, s, wq=wq, s_ch=sch, workspace=ws)
    times = []
    for _ in range(max(1, args.steps)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        w8.w8a8_gptq_quantize(w, x, s, wq=wq, s_ch=sch, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    t = statistics.median(times)
    flops = {"hessian": T * K * (K + 1), "cholesky": K ** 3 / 3, "inverse": K ** 3 / 3,
             "quantize": N * K * K}
    total = sum(flops.values())
    peak = measure_f64_peak()
    return {"case": args.case, "ms_per_call": round(t * 1e3, 3),
            "fp64_tflops": round(total / t / 1e12, 2), "fp64_peak_tflops_measured": round(peak, 2),
            "frac": round(total / t / 1e12 / peak, 4),
            "flops": {k: float(v) for k, v in flops.items()},
            "note": "median of K calls; each call synchronizes (offline preparation)"}


def run_case(args):
    """`--case gemm:M:N:K[:variant[:ctas[:tile_n]]]` (INT8; ctas and tile_n as in
    w8a8_gemm_dequant_ex), `gemm8:M:N:K[:variant[:ctas[:tile_n]]]` (FP8), `rms:M:K`, `rmsres:M:K`, `quant:M:K`, `static:M:K` or
    `silu:M:I`:
    one kernel launched repeatedly (a CUDA graph of back-to-back launches)."""
    import int8_w8a8_quantized_smoothed_b200 as w8
    from int8_w8a8_quantized_smoothed_b200 import build as wbuild, synth
    wbuild.build()
    parts = args.case.split(":")
    dev = torch.device("cuda", 0)
    if parts[0] == "gptq":
        return run_gptq_case(args, [int(v) for v in parts[1:4]])
    if parts[0] == "silug":
        # the fused gate|up GEMM + SiLU*up + quantization call, silug:M:I:K
        M, I, K = (int(v) for v in parts[1:4])
        copies = max(1, math.ceil(4 * 126e6 / (2 * I * K)))
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev)
        st = torch.rand(M, device=dev) * 1e-2
        ws_ = [torch.randint(-127, 128, (2 * I, K), dtype=torch.int8, device=dev)
               for _ in range(copies)]
        sc = torch.rand(2 * I, device=dev) * 1e-3
        a = torch.empty(M, I, dtype=torch.float32, device=dev)
        q = torch.empty(M, I, dtype=torch.int8, device=dev)
        s_out = torch.empty(M, dtype=torch.float32, device=dev)
        wsp = w8.Workspace(dev)

        def launch(i):
            w8.w8a8_gemm_silu_quant(xq, st, ws_[i % copies], sc, a=a, q=q, s_out=s_out,
                                    workspace=wsp)
        work = gemm_bytes(M, 2 * I, K) - 2 * M * 2 * I + 5 * M * I + 4 * M
        flops = 2 * M * 2 * I * K
    elif parts[0] in ("gemm", "gemm8"):
        M, N, K = (int(v) for v in parts[1:4])
        variant = int(parts[4]) if len(parts) > 4 else 0
        ctas = int(parts[5]) if len(parts) > 5 else 0
        tile_n = int(parts[6]) if len(parts) > 6 else 0
        fp8 = parts[0] == "gemm8"
        copies = max(1, math.ceil(4 * 126e6 / (N * K)))  # rotate weights through > 4x L2

        def codes(shape):
            if not fp8:
                return torch.randint(-127, 128, shape, dtype=torch.int8, device=dev)
            c = torch.randint(0, 256, shape, dtype=torch.uint8, device=dev)
            c[(c & 0x7F) == 0x7F] = 0x30  # no NaN codes
            return c.view(w8.FP8)
        xq = codes((M, K))
        st = torch.rand(M, device=dev) * 1e-2
        ws_ = [codes((N, K)) for _ in range(copies)]
        sc = torch.rand(N, device=dev) * 1e-3
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        wsp = w8.Workspace(dev)
        gemm = w8.w8a8_gemm_dequant_fp8 if fp8 else w8.w8a8_gemm_dequant_ex

        def launch(i):
            gemm(xq, st, ws_[i % copies], sc, y=y, workspace=wsp, variant=variant, ctas=ctas,
                 tile_n=tile_n)
        work = gemm_bytes(M, N, K)
        flops = 2 * M * N * K
    else:
        # row kernels: rms:M:K, rmsres:M:K, quant:M:K, silu:M:I; inputs rotate over enough
        # copies to exceed L2
        kind, M, K = parts[0], int(parts[1]), int(parts[2])
        cols = 2 * K if kind == "silu" else K
        copies = max(1, math.ceil(4 * 126e6 / (M * cols * 2)))
        xs = [synth.activation_device(M, cols, 1 + c, dev) for c in range(copies)]
        res = synth.activation_device(M, K, 99, dev)
        h = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        g = torch.ones(K, device=dev)
        q = torch.empty(M, K, dtype=torch.int8, device=dev)
        s = torch.empty(M, device=dev)

        def launch(i):
            x = xs[i % copies]
            if kind == "rms":
                w8.w8a8_smooth_rmsnorm_quant(x, g, EPS, q=q, s_tok=s)
            elif kind == "rmsres":
                w8.w8a8_smooth_rmsnorm_quant(x, g, EPS, residual=res, h_out=h, q=q, s_tok=s)
            elif kind == "quant":
                w8.w8a8_quantize_rows(x, g, q=q, s_tok=s)
            elif kind == "static":
                w8.w8a8_quantize_rows_static(x, 0.05, g, q=q, s_tok=s)
            else:
                w8.w8a8_silu_mul_quant(x, q=q, s_tok=s)
        work = {"rms": 3 * M * K, "rmsres": 7 * M * K, "quant": 3 * M * K, "static": 3 * M * K,
                "silu": 5 * M * K}[kind] + 4 * M + 4 * K
    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize()
    # time a CUDA graph of `steps` launches, so launch gaps of short kernels do not count
    cg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cg, capture_error_mode="thread_local"):
        for i in range(args.steps):
            launch(i)
    cg.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    cg.replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / args.steps
    out = {"case": args.case, "us_per_launch": round(t * 1e6, 3),
           "GBps_algorithmic": round(work / t / 1e9, 1),
           "note": "CUDA graph of back-to-back launches"}
    if parts[0] in ("gemm", "gemm8", "silug"):
        out["TOPS"] = round(flops / t / 1e12, 1)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode8b")
    ap.add_argument("--extra", default=None,
                    help="comma-separated further workloads measured in the same run and "
                         "reported as nested records of the line (default: prefill8b with the "
                         "decode8b workload, else none; 'none' disables)")
    ap.add_argument("--case", default=None)
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the dominant kernel, if measured")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="gate|up GEMM and SiLU*up+quant as separate launches instead of the "
                         "fused SiLU*up epilogue")
    ap.add_argument("--o-norm-one-launch", action="store_true",
                    help="the residual RMSNorm + quant in the o GEMM's row tail at M <= 64 "
                         "(w8a8_gemm_rmsnorm_quant one_launch) instead of a second launch")
    ap.add_argument("--fused-block", action="store_true",
                    help="run each decoder block's linear path as the single fused persistent "
                         "kernel (w8a8_block_decode; M <= 64)")
    ap.add_argument("--fp8", action="store_true",
                    help="the FP8 (E4M3) variant of the path: FP8 row kernels and GEMMs")
    ap.add_argument("--overlap", type=int, choices=[0, 1, 2], default=2,
                    help="kernel overlap mode (w8a8_set_overlap); 2 = dependent launch with "
                         "static-weight prefetch")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.case is None:
        ap.error("--warmup must be at least 3")
    if args.fp8 and args.fused_block:
        ap.error("the fused block kernel (--fused-block) has INT8 codes only")
    if args.extra is None:
        args.extra = "prefill8b" if (args.workload == "decode8b" and not args.fused_block) \
            else "none"
    for e in args.extra.split(","):
        if e not in WORKLOADS and e not in ("", "none"):
            ap.error(f"--extra: unknown workload {e}")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0
    if args.case:
        print(json.dumps(run_case(args)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    out = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
