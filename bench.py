"""Benchmark of the B200 LiquidQuant W4A8 GEMM path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|mlp_up|down_sweep|tiny]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

One step is one pass of the per-forward hot path over one batch: for every
token count M of the workload, per-token INT8 quantization of the bf16
activations followed by the W4A8 GEMM against a layer's packed weights (the
weights are quantized offline, once, as in the method).  The default workload
is the decode attention-projection layer, N = K = 4096, M in {1, 4, 16}.

Timing: K steps are captured in one CUDA graph and replayed once between CUDA
events on the launching stream, after W warm-up steps and about a second of
untimed replays (so the clock sampler sees the GPU under load).  Each GEMM
launch reads a different copy of the layer's packed weights, rotating over
enough copies that the working set is several times the 126 MB L2, so every
launch streams its weights from HBM.  The GEMM's own duration per launch (the
roofline's denominator) comes from a second graph of K back-to-back GEMM calls
per M, timed the same way: the launches overlap through programmatic dependent
launch exactly as in the step, and replay time / K is the time per launch.

The end-to-end variant (`e2e`) runs the same step through the same calls
with host buffers: each batch's bf16 rows are read from pinned host memory by
the activation quantizer and each GEMM writes its outputs to pinned host
memory, both directly over the host link (zero-copy I/O of the library), so
the transfers sit inside the timed region without copy nodes that would end
the programmatic-launch chain.  Where the device cannot address the pinned
buffers, it copies instead (one copy in, one copy out per step).

The default (decode) run also measures, in the same process: the prefill
layer, a dense INT8 ceiling (torch._int_mm at 8192^3), the MLP up/gate layer
and the down-projection sweep (every M of both), the fused SwiGLU gate/up pair
against two GEMMs plus a separate activation, the grouped GEMM, the
dequantization ablation and the W4 x FP8 variant -- each as side objects of
the JSON line.

With --gpus N > 1 (launched by torchrun) every rank runs an independent
replica (the path has no exchange step); the time is the max over ranks and
the value the sum of all ranks' work.

Prints ONE JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import platform
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio: 4.5 PFLOP/s int8 vs 2.25 bf16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "mlp_up", "down_sweep", "tiny"])
    ap.add_argument("--soak-s", type=float, default=1.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the prefill measurement of the default run")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# workload accounting
# ---------------------------------------------------------------------------

def gemm_bytes(M, N, K, G=64):
    """Algorithmic HBM bytes of one GEMM: packed u4 weights, u8 scale and offset,
    fp32 channel scales, int8 activations, fp32 token scales, bf16 output."""
    return N * K // 2 + 2 * N * (K // G) + 4 * N + M * K + 4 * M + 2 * M * N


def linear_bytes(M, N, K, G=64):
    """Algorithmic HBM bytes of one activation-quantization + GEMM pass: the
    weights, bf16 activations in and bf16 output (the INT8 codes and token scales
    are intermediates; the fused launch never writes them)."""
    return N * K // 2 + 2 * N * (K // G) + 4 * N + 2 * M * K + 2 * M * N


def step_accounting(w):
    gb = sum(linear_bytes(M, w.N, w.K) for M in w.Ms)
    ops = sum(2 * M * w.N * w.K for M in w.Ms)
    return gb, 0, ops


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "w4a8_bit_weight_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_source") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_gemm_launch")


def reduce_max(value: float, world: int, device) -> float:
    """Max of `value` over all ranks (the slowest rank sets the job's time)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.proc = None
        self.lines = []
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if gpu_uuid:
            cmd += ["-i", gpu_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if ts < t0 or ts > t1:
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# the CPU baseline: the oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------

def cpu_baseline(w, budget_s=10.0):
    import oracle
    from w4a8_bit_weight_b200 import synth
    X, W = synth.make_workload(w)
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    xb = synth.bf16_bits(X)
    gb, ab, ops = step_accounting(w)
    Ms = list(w.Ms)
    # prefill-size layers: a bounded sample of token rows per step
    rows = {M: min(M, 64) for M in Ms}
    frac = sum(rows.values()) / sum(Ms)
    t0 = time.perf_counter()
    steps = 0
    while True:
        for M in Ms:
            xq, sx = oracle.quantize_act(xb[:rows[M]])
            oracle.w4a8_gemm(xq, sx, o_qw, o_s, o_a, o_sc)
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    sample = (f"{steps} oracle steps, each quantize_act + w4a8_gemm (dequant, int64 contraction, "
              f"epilogue) for M in {Ms}" + ("" if frac == 1 else f" with min(M,64) token rows") +
              f", N={w.N}, K={w.K}; {el:.1f} s")
    # throughput in the same unit: the step's algorithmic bytes, scaled to the rows sampled
    byts = sum(linear_bytes(rows[M], w.N, w.K) for M in Ms)
    cores = oracle.num_threads()
    # the same on one core, for a shorter sample
    oracle.set_num_threads(1)
    t1 = time.perf_counter()
    steps1 = 0
    try:
        while True:
            for M in Ms:
                xq, sx = oracle.quantize_act(xb[:rows[M]])
                oracle.w4a8_gemm(xq, sx, o_qw, o_s, o_a, o_sc)
            steps1 += 1
            el1 = time.perf_counter() - t1
            if el1 >= budget_s / 3:
                break
    finally:
        oracle.set_num_threads(cores)
    return {"value": byts * steps / el / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle", "sample": sample,
            "tops": 2 * sum(rows[M] for M in Ms) * w.N * w.K * steps / el / 1e12,
            "value_1core": byts * steps1 / el1 / 1e9, "sample_1core": f"{steps1} steps on one thread, {el1:.1f} s",
            "host": host_cpu()}


def host_cpu():
    """The host's CPU model and logical CPU count (for the oracle timings)."""
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


# ---------------------------------------------------------------------------
# our path
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    Ms = list(w.Ms)
    gb, ab, ops = step_accounting(w)
    step_bytes = gb + ab

    X, W = synth.make_workload(w)
    qw, s_u8, a_u8, s_c = lq.lq_quantize_weights(W.to(dev))
    wset_bytes = qw.numel() + s_u8.numel() + a_u8.numel() + 4 * s_c.numel()
    n_sets = max(4, int(np.ceil(3 * L2_BYTES / wset_bytes)))
    n_sets = min(n_sets, 64)
    sets = [(qw, s_u8, a_u8, s_c)] + [(qw.clone(), s_u8.clone(), a_u8.clone(), s_c.clone())
                                      for _ in range(n_sets - 1)]
    Xd = X.to(dev)
    Mx = max(Ms)
    xq_buf = {M: torch.empty(M, w.K, dtype=torch.int8, device=dev) for M in Ms}
    sx_buf = {M: torch.empty(M, dtype=torch.float32, device=dev) for M in Ms}
    # the outputs of all M of a step are row ranges of one buffer (one copy back per step)
    out_all = torch.empty(sum(Ms), w.N, dtype=torch.bfloat16, device=dev)
    out_off = {M: sum(Ms[:i]) for i, M in enumerate(Ms)}
    out_buf = {M: out_all[out_off[M]:out_off[M] + M] for M in Ms}
    ws_need = max(lq.lq_w4a8_gemm_workspace_size(M, w.N, w.K) for M in Ms)
    ws = torch.zeros(max(ws_need, 16), dtype=torch.uint8, device=dev)
    # lq_w4a8_linear's workspace, for its side measurement (fused vs two launches)
    lin_ws_need = max(lq.lq_w4a8_linear_workspace_size(M, w.N, w.K, lq.LINEAR_TWO_LAUNCHES) for M in Ms)
    ws_lin = torch.zeros(max(lin_ws_need, 16), dtype=torch.uint8, device=dev)
    # pinned host buffers for the end-to-end variant.  The library reads activations from and
    # writes outputs to pinned host memory directly (zero-copy I/O, lq.h): the step's
    # quantizers read their rows of X_host over the host link and its GEMMs write their rows
    # of out_host.  Where the device cannot address them at the same pointer, the variant
    # copies instead: the step's batches are the first M rows of one token set, so one copy
    # of the first max(M) rows brings all of its inputs, and one copy takes all outputs back.
    X_host = X.pin_memory()
    out_host = torch.empty(sum(Ms), w.N, dtype=torch.bfloat16).pin_memory()
    out_host_buf = {M: out_host[out_off[M]:out_off[M] + M] for M in Ms}
    zero_copy = lq.lq_device_addressable(X_host) and lq.lq_device_addressable(out_host)
    Xd_e2e = None if zero_copy else torch.empty_like(Xd)

    stream = torch.cuda.Stream(dev)
    counter = [0]

    def step(e2e=False):
        if e2e and not zero_copy:
            Xd_e2e[:Mx].copy_(X_host[:Mx], non_blocking=True)
        for M in Ms:
            src = (X_host[:M] if zero_copy else Xd_e2e[:M]) if e2e else Xd[:M]
            lq.lq_quantize_act(src, out=(xq_buf[M], sx_buf[M]))
            wq = sets[counter[0] % n_sets]
            counter[0] += 1
            dst = out_host_buf[M] if (e2e and zero_copy) else out_buf[M]
            lq.lq_w4a8_gemm(xq_buf[M], sx_buf[M], *wq, out=dst, workspace_buf=ws)
        if e2e and not zero_copy:
            out_host.copy_(out_all, non_blocking=True)

    def capture(nsteps, e2e=False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(nsteps):
                step(e2e)
        return g

    def capture_gemms(M, n):
        """n back-to-back GEMMs of one M, the weights rotating over the L2-cold copies."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                lq.lq_w4a8_gemm(xq_buf[M], sx_buf[M], *sets[i % n_sets], out=out_buf[M], workspace_buf=ws)
        return g

    lin_paths = {"fused": lq.LINEAR_FUSED, "two_launches": lq.LINEAR_TWO_LAUNCHES}
    n_lin = min(args.steps, 100)

    def capture_linear(M, path):
        """n_lin back-to-back lq_w4a8_linear calls of one M on one path (None if it does not apply)."""
        if path == lq.LINEAR_FUSED and lq.lq_w4a8_linear_workspace_size(M, w.N, w.K, path) != 0:
            return None
        for i in range(2):
            lq.lq_w4a8_linear(Xd[:M], *sets[i % n_sets], out=out_buf[M], workspace_buf=ws_lin, path=path)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_lin):
                lq.lq_w4a8_linear(Xd[:M], *sets[i % n_sets], out=out_buf[M], workspace_buf=ws_lin, path=path)
        return g

    with torch.cuda.stream(stream):
        # warm-up, eager, W steps (first launches also load the kernels)
        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize(dev)
        st = lq.lq_get_device_error(dev)
        if st != 0:
            raise RuntimeError(f"device error after warm-up: {st}")
        g_timed = capture(args.steps)
        g_gemm = {M: capture_gemms(M, args.steps) for M in Ms}
        g_lin = {} if args.no_secondary else {(M, k): capture_linear(M, p) for M in Ms for k, p in lin_paths.items()}
        g_e2e = None if args.no_e2e else capture(args.steps, e2e=True)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    time.sleep(0.3)
    t_load0 = time.time()
    # Every timed graph is replayed once untimed first (its first launch also
    # uploads it to the device), then an untimed soak of the step graph so the
    # clocks settle and the sampler sees load.
    with torch.cuda.stream(stream):
        for g in [g_timed, *g_gemm.values(), *[x for x in g_lin.values() if x is not None]] + (
                [g_e2e] if g_e2e is not None else []):
            g.replay()
        torch.cuda.synchronize(dev)
        soak_end = time.time() + args.soak_s
        while time.time() < soak_end:
            g_timed.replay()
            torch.cuda.synchronize(dev)

    def timed(graph):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return reduce_max(e0.elapsed_time(e1), world, dev)

    with torch.cuda.stream(stream):
        ms_total = timed(g_timed)
        # the dominant kernel on its own: K back-to-back GEMMs per M in one graph
        # (the launches overlap through programmatic dependent launch as they do
        # in the step); its duration per launch is the replay time / K
        gemm_ms = {M: timed(g_gemm[M]) / args.steps for M in Ms}
        ms_e2e = timed(g_e2e) if g_e2e is not None else None
        lin_us = {key: (1e3 * timed(g) / n_lin if g is not None else None) for key, g in g_lin.items()}
    t_load1 = time.time()
    clocks = sampler.stop(t_load0, t_load1) if sampler else None
    st = lq.lq_get_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {st}")

    K_ = args.steps
    value = world * step_bytes * K_ / (ms_total * 1e-3) / 1e9
    # dominant kernel: the GEMM, one launch of each M
    per_M = {M: float(t) for M, t in gemm_ms.items()}
    gemm_time_s = sum(per_M.values()) * 1e-3
    gemm_bytes_total = sum(gemm_bytes(M, w.N, w.K) for M in Ms)
    achieved = gemm_bytes_total / gemm_time_s / 1e9
    pk, pk_src = peaks()
    hbm_peak = float(pk["hbm_gbs"])
    int8_peak = INT8_OVER_BF16 * float(pk["bf16_tflops"])
    gemm_launches = args.steps * len(Ms)
    n_traffic = ncu_traffic(args.workload)
    res = {
        "metric": "W4A8 GEMM TOPS and HBM GB/s vs roofline at decode M=1-16 and prefill M=4096",
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K_,
        "warmup": args.warmup,
        "ms_per_step": ms_total / K_,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded N(0,1) activations with outlier channels, N(0,0.02) weights)",
        "config": {
            "workload": w.note, "M": Ms, "N": w.N, "K": w.K, "group": 64,
            "step": "per M: lq_quantize_act + lq_w4a8_gemm (weights quantized offline)",
            "l2": f"weights rotate over {n_sets} copies ({n_sets * wset_bytes / 2**20:.0f} MiB > 126 MB L2)",
            "timing": "one CUDA graph of K steps between CUDA events; kernels launched with "
                      "programmatic dependent launch",
            "parallelism": f"replicas x{world}",
        },
        "tops": world * ops * K_ / (ms_total * 1e-3) / 1e12,
        "gpu_launches": K_ * 2 * len(Ms),
        "roofline": {
            "bound": "hbm", "kernel": "w4a8_gemm_kernel", "achieved": achieved, "peak": hbm_peak,
            "unit": "GB/s", "frac": achieved / hbm_peak,
            "frac_of_8000_gbs": achieved / 8000.0,  # against the HBM3e figure the targets are stated on
            "traffic": n_traffic,
            "peak_source": pk_src,
            "per_launch_us": {str(M): 1e3 * t for M, t in per_M.items()},
            "launches": gemm_launches,
            "how": "per M, K back-to-back lq_w4a8_gemm calls (weights rotating over the L2-cold "
                   "copies) in one CUDA graph between CUDA events, right after the timed step "
                   "replay; duration per launch = replay time / K",
            "bytes_per_launch": {str(M): gemm_bytes(M, w.N, w.K) for M in Ms},
        },
        "clocks": clocks,
    }
    if ms_e2e is not None:
        h2d = (sum(Ms) if zero_copy else max(Ms)) * w.K * 2
        d2h = sum(Ms) * w.N * 2
        res["e2e"] = {"value": world * step_bytes * K_ / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": ms_e2e / K_,
                      "how": ("per step and M: lq_quantize_act reads the batch's bf16 rows from pinned host "
                              "memory and lq_w4a8_gemm writes its bf16 outputs to pinned host memory, both "
                              "directly over the host link (zero-copy I/O); same CUDA graph method"
                              if zero_copy else
                              "per step: one pinned host -> device copy of the activation rows (every "
                              "batch of the step is a prefix of them), quantize_act + gemm per M, one device -> "
                              "pinned host copy of all outputs; same CUDA graph method")}
    if lin_us:
        res["linear"] = {
            "what": "lq_w4a8_linear (activation quantization + GEMM) per M, one fused launch vs the "
                    "two launches, each as back-to-back calls of one M in one CUDA graph; us per call",
            **{str(M): {"fused_us": lin_us[(M, "fused")], "two_launches_us": lin_us[(M, "two_launches")],
                        "auto_path": "fused" if lq.lq_w4a8_linear_workspace_size(M, w.N, w.K) == 0
                        else "two_launches"} for M in Ms}}
    res["int8_peak_tops"] = int8_peak
    if args.workload == "decode" and not args.no_secondary:
        ceil = int8_ceiling(dev)
        res["int8_ceiling"] = ceil
        pre = secondary_workload("prefill", dev)
        g = pre["4096"]
        pre["roofline"] = {"bound": "tensor", "kernel": "w4a8_gemm_pair_kernel", "achieved": g["gemm_tops"],
                           "peak": int8_peak, "unit": "TOPS", "frac": g["gemm_tops"] / int8_peak,
                           "peak_source": f"{pk_src}: {INT8_OVER_BF16:g} x bf16 burst",
                           "frac_of_nominal_4500": g["gemm_tops"] / 4500.0,
                           "traffic": ncu_traffic("prefill")}
        if "tops" in ceil:
            pre["roofline"]["measured_int8_ceiling_tops"] = ceil["tops"]
            pre["roofline"]["frac_of_measured_int8_ceiling"] = g["gemm_tops"] / ceil["tops"]
        res["prefill"] = pre
        res["mlp_up"] = shape_sweep("mlp_up", dev, hbm_peak, int8_peak)
        res["down_sweep"] = shape_sweep("down_sweep", dev, hbm_peak, int8_peak)
        res["swiglu"] = swiglu_side(dev, hbm_peak, int8_peak)
        res["grouped"] = grouped_side(dev, int8_peak, hbm_peak)
        res["ablation"] = ablation_side(dev, hbm_peak)
        try:
            res["w4f8"] = w4f8_side(dev, hbm_peak)
        except Exception as ex:  # a side measurement never takes the bench line down
            res["w4f8"] = {"error": str(ex)[:200]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w)
    return res


def grouped_side(dev, int8_peak, hbm_peak, n=20):
    """The grouped GEMM on a mixture-of-experts layer: 8 experts of the MLP up/gate
    geometry (N=14336, K=4096), tokens routed top-2 by a seeded random assignment;
    a decode batch (16 tokens -> 32 rows) and a prefill batch (4096 tokens -> 8192
    rows).  n back-to-back grouped GEMMs in one CUDA graph between CUDA events.
    The experts are one seeded expert quantized once and copied 8 times (separate
    memory, so every expert's bytes are read from HBM; the values do not change
    the timing)."""
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth
    E, N, K = 8, 14336, 4096
    w = synth.WORKLOADS["mlp_up"]
    X, W = synth.make_workload(w)
    qw, s_u8, a_u8, s_c = lq.lq_quantize_weights(W.to(dev))
    qw_all = torch.cat([qw] * E)
    s_all = torch.cat([s_u8] * E, dim=1).contiguous()
    a_all = torch.cat([a_u8] * E, dim=1).contiguous()
    sc_all = torch.cat([s_c] * E)
    del qw, s_u8, a_u8, s_c
    rng = np.random.default_rng(11)
    stream = torch.cuda.Stream(dev)
    res = {"workload": "mixture-of-experts up/gate layer: 8 experts N=14336 K=4096, top-2 routing",
           "how": f"{n} back-to-back lq_w4a8_grouped_gemm calls in one CUDA graph between CUDA events"}
    Xd = X.to(dev)
    for name, tokens in (("decode", 16), ("prefill", 4096)):
        rows = 2 * tokens
        sizes = np.bincount(rng.integers(0, E, size=rows), minlength=E)
        m_off = torch.from_numpy(np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)).to(dev)
        src = Xd[torch.arange(rows, device=dev) % Xd.shape[0]]
        xq, sx = lq.lq_quantize_act(src)
        out = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
        with torch.cuda.stream(stream):
            for _ in range(3):
                lq.lq_w4a8_grouped_gemm(xq, sx, qw_all, s_all, a_all, sc_all, m_off, N, out=out)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(n):
                    lq.lq_w4a8_grouped_gemm(xq, sx, qw_all, s_all, a_all, sc_all, m_off, N, out=out)
            g.replay()
            torch.cuda.synchronize(dev)
            ts = []
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ts.append(e0.elapsed_time(e1) / n)
        if lq.lq_get_device_error(dev) != 0:
            raise RuntimeError("device error in the grouped measurement")
        t_ms = sorted(ts)[1]
        experts = int((sizes > 0).sum())
        byts = experts * (N * K // 2 + 2 * N * K // 64 + 4 * N) + rows * K + 4 * rows + 2 * rows * N
        ops = 2 * rows * N * K
        gbs = byts / (t_ms * 1e-3) / 1e9
        tops = ops / (t_ms * 1e-3) / 1e12
        res[name] = {"rows": rows, "experts_used": experts, "us": 1e3 * t_ms, "gbs": gbs, "tops": tops,
                     "frac_of_hbm": gbs / hbm_peak, "frac_of_int8": tops / int8_peak}
        del xq, sx, out, src, g
    return res


def ablation_side(dev, hbm_peak, n=40):
    """The pages' ablation of the dequantization arithmetic and pipeline, redone on the
    tile kernel: SWAR (LQQ) vs per-element expansion, A in tensor memory (implicit
    pipeline) vs a shared-memory A tile (explicit pipeline).  A decode layer (16 tokens,
    N = K = 4096, 16-token tiles) and a down-projection at 64 tokens (N = 4096,
    K = 14336, 64-token tiles), both in 4-CTA clusters; n back-to-back launches per
    variant in one CUDA graph, the weights rotating over L2-cold copies."""
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth
    names = {lq.ABL_IMPLICIT: "lqq_implicit", lq.ABL_NAIVE: "naive_implicit", lq.ABL_EXPLICIT: "lqq_explicit",
             lq.ABL_NAIVE_EXPLICIT: "naive_explicit"}
    res = {"how": f"{n} back-to-back lq_w4a8_gemm_ablation calls per variant in one CUDA graph; us per launch",
           "variants": "lqq = SWAR IMAD+XOR expansion, naive = one weight at a time; implicit = A in TMEM, "
                       "explicit = A tile in shared memory"}
    stream = torch.cuda.Stream(dev)
    for label, (M, N, K, bt) in (("decode_16x4096x4096", (16, 4096, 4096, 16)),
                                 ("down_64x4096x14336", (64, 4096, 14336, 64))):
        X, W = synth.make_problem(M, N, K, seed=21, n_outliers=8)
        qw, s_u8, a_u8, s_c = lq.lq_quantize_weights(W.to(dev))
        wset = qw.numel() + 2 * s_u8.numel() + 4 * s_c.numel()
        n_sets = min(48, max(4, int(np.ceil(3 * L2_BYTES / wset))))
        sets = [(qw, s_u8, a_u8, s_c)] + [(qw.clone(), s_u8.clone(), a_u8.clone(), s_c.clone())
                                          for _ in range(n_sets - 1)]
        xq, sx = lq.lq_quantize_act(X.to(dev))
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        entry = {}
        with torch.cuda.stream(stream):
            for v, nm in names.items():
                for i in range(2):
                    lq.lq_w4a8_gemm_ablation(xq, sx, *sets[i % n_sets], v, bt, out=out)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for i in range(n):
                        lq.lq_w4a8_gemm_ablation(xq, sx, *sets[i % n_sets], v, bt, out=out)
                g.replay()
                torch.cuda.synchronize(dev)
                ts = []
                for _ in range(3):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                    torch.cuda.synchronize(dev)
                    ts.append(1e3 * e0.elapsed_time(e1) / n)
                us = sorted(ts)[1]
                gbs = gemm_bytes(M, N, K) / (us * 1e-6) / 1e9
                entry[nm] = {"us": us, "gbs": gbs, "frac_of_hbm": gbs / hbm_peak}
                del g
        if lq.lq_get_device_error(dev) != 0:
            raise RuntimeError("device error in the ablation measurement")
        base = entry["lqq_implicit"]["us"]
        for nm in entry:
            entry[nm]["slowdown_vs_lqq_implicit"] = entry[nm]["us"] / base
        res[label] = entry
        del sets, qw, s_u8, a_u8, s_c
    return res


def w4f8_side(dev, hbm_peak, n=40):
    """The W4 x FP8 variant on the decode layer (N = K = 4096, M = 1, 4, 16): n back-to-back
    lq_w4f8_gemm calls per M in one CUDA graph, weights rotating over L2-cold copies."""
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth
    w = synth.WORKLOADS["decode"]
    X, W = synth.make_workload(w)
    qw4, s_w = lq.lq_quantize_weights_w4(W.to(dev))
    wset = qw4.numel() + 4 * s_w.numel()
    n_sets = min(48, max(4, int(np.ceil(3 * L2_BYTES / wset))))
    sets = [(qw4, s_w)] + [(qw4.clone(), s_w.clone()) for _ in range(n_sets - 1)]
    stream = torch.cuda.Stream(dev)
    res = {"workload": w.note, "how": f"{n} back-to-back lq_w4f8_gemm calls per M in one CUDA graph; "
                                      "bytes = INT4 weights + s_w + e4m3 x + s_x + bf16 out"}
    Xd = X.to(dev)
    for M in w.Ms:
        x_f8, s_x = lq.lq_quantize_act_f8(Xd[:M])
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
        with torch.cuda.stream(stream):
            for i in range(2):
                lq.lq_w4f8_gemm(x_f8, s_x, *sets[i % n_sets], out=out)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    lq.lq_w4f8_gemm(x_f8, s_x, *sets[i % n_sets], out=out)
            g.replay()
            torch.cuda.synchronize(dev)
            ts = []
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ts.append(1e3 * e0.elapsed_time(e1) / n)
        if lq.lq_get_device_error(dev) != 0:
            raise RuntimeError("device error in the W4 x FP8 measurement")
        us = sorted(ts)[1]
        byts = w.N * w.K // 2 + 4 * w.N + M * w.K + 4 + 2 * M * w.N
        res[str(M)] = {"us": us, "gbs": byts / (us * 1e-6) / 1e9, "frac_of_hbm": byts / (us * 1e-6) / 1e9 / hbm_peak}
        del g
    return res


def _graph_us(stream, dev, fn, n, reps=3):
    """Median over `reps` replays of a CUDA graph of n calls of fn(i), us per call
    (the graph is replayed once untimed first: its first launch also uploads it)."""
    for i in range(2):
        fn(i)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fn(i)
    g.replay()
    torch.cuda.synchronize(dev)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(1e3 * e0.elapsed_time(e1) / n)
    del g
    return sorted(ts)[len(ts) // 2]


def _roofline(M, N, K, us, hbm_peak, int8_peak):
    byts = gemm_bytes(M, N, K)
    ops = 2.0 * M * N * K
    t_hbm, t_tc = byts / (hbm_peak * 1e9), ops / (int8_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    return {"us": us, "gbs": byts / (us * 1e-6) / 1e9, "tops": ops / (us * 1e-6) / 1e12, "bound": bound,
            "frac": max(t_hbm, t_tc) / (us * 1e-6)}


def shape_sweep(workload, dev, hbm_peak, int8_peak, n=20):
    """Back-to-back lq_w4a8_gemm launches of each M of a workload (its N, K, seeded
    weights and activations), weights rotating over L2-cold copies; us per launch,
    GB/s of algorithmic bytes, TOPS, and the fraction of the larger of the HBM time
    and the INT8 tensor time."""
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth
    w = synth.WORKLOADS[workload]
    X, W = synth.make_workload(w)
    qw, s_u8, a_u8, s_c = lq.lq_quantize_weights(W.to(dev))
    wset = qw.numel() + 2 * s_u8.numel() + 4 * s_c.numel()
    n_sets = min(48, max(4, int(np.ceil(3 * L2_BYTES / wset))))
    sets = [(qw, s_u8, a_u8, s_c)] + [(qw.clone(), s_u8.clone(), a_u8.clone(), s_c.clone())
                                      for _ in range(n_sets - 1)]
    stream = torch.cuda.Stream(dev)
    res = {"workload": w.note, "how": f"{n} back-to-back lq_w4a8_gemm calls per M in one CUDA graph, "
                                      f"weights rotating over {n_sets} copies; roofline = max(HBM time at "
                                      f"{hbm_peak:.0f} GB/s, INT8 time at {int8_peak:.0f} TOPS)"}
    Xd = X.to(dev)
    for M in w.Ms:
        xq, sx = lq.lq_quantize_act(Xd[:M])
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
        with torch.cuda.stream(stream):
            us = _graph_us(stream, dev, lambda i: lq.lq_w4a8_gemm(xq, sx, *sets[i % n_sets], out=out), n)
        res[str(M)] = _roofline(M, w.N, w.K, us, hbm_peak, int8_peak)
        del xq, sx, out
    if lq.lq_get_device_error(dev) != 0:
        raise RuntimeError(f"device error in the {workload} sweep")
    return res


def swiglu_side(dev, hbm_peak, int8_peak, n=20):
    """The MLP up/gate layer as a gated FFN pair: F = 14336 gate + 14336 up channels,
    K = 4096, M = 16 / 256 / 4096.  One lq_w4a8_gemm_swiglu launch on the interleaved
    [2F, K] weights against two lq_w4a8_gemm launches (gate, up) plus the separate
    activation silu(gate) * up (torch, bf16) -- the same work, unfused."""
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth
    w = synth.WORKLOADS["mlp_up"]
    F, K = w.N, w.K
    X, W = synth.make_problem(max(w.Ms), 2 * F, K, seed=31, n_outliers=41)
    qw, s_u8, a_u8, s_c = lq.lq_quantize_weights(W.to(dev))
    # gate rows are the even rows, up rows the odd ones: the same weights, unfused
    qg, sg, ag, cg = lq.lq_quantize_weights(W[0::2].contiguous().to(dev))
    qu, su, au, cu = lq.lq_quantize_weights(W[1::2].contiguous().to(dev))
    wset = 2 * (qw.numel() + 2 * s_u8.numel() + 4 * s_c.numel())
    n_sets = min(16, max(2, int(np.ceil(3 * L2_BYTES / wset))))
    fused = [(qw, s_u8, a_u8, s_c)] + [(qw.clone(), s_u8.clone(), a_u8.clone(), s_c.clone()) for _ in range(n_sets - 1)]
    split = [((qg, sg, ag, cg), (qu, su, au, cu))] + [
        ((qg.clone(), sg.clone(), ag.clone(), cg.clone()), (qu.clone(), su.clone(), au.clone(), cu.clone()))
        for _ in range(n_sets - 1)]
    stream = torch.cuda.Stream(dev)
    res = {"workload": f"gated FFN up/gate pair F={F} (+{F}) K={K}, interleaved weights",
           "how": f"{n} back-to-back calls per M in one CUDA graph, weights rotating over {n_sets} copies; "
                  "unfused = gate GEMM + up GEMM + torch silu(g)*u on their bf16 outputs"}
    Xd = X.to(dev)
    for M in w.Ms:
        xq, sx = lq.lq_quantize_act(Xd[:M])
        out = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
        g_out = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
        u_out = torch.empty(M, F, dtype=torch.bfloat16, device=dev)

        def unfused(i):
            gw, uw = split[i % n_sets]
            lq.lq_w4a8_gemm(xq, sx, *gw, out=g_out)
            lq.lq_w4a8_gemm(xq, sx, *uw, out=u_out)
            torch.mul(torch.nn.functional.silu(g_out), u_out, out=out)

        with torch.cuda.stream(stream):
            us_f = _graph_us(stream, dev, lambda i: lq.lq_w4a8_gemm_swiglu(xq, sx, *fused[i % n_sets], out=out), n)
            us_u = _graph_us(stream, dev, unfused, n)
        r = _roofline(M, 2 * F, K, us_f, hbm_peak, int8_peak)
        # the fused output is F columns, not 2F: count its bytes as written
        byts = gemm_bytes(M, 2 * F, K) - 2 * M * F
        r["gbs"] = byts / (us_f * 1e-6) / 1e9
        res[str(M)] = {"fused_us": us_f, "unfused_us": us_u, "speedup": us_u / us_f, "fused": r}
        del xq, sx, out, g_out, u_out
    if lq.lq_get_device_error(dev) != 0:
        raise RuntimeError("device error in the SwiGLU measurement")
    return res


def int8_ceiling(dev, size=8192, n=10):
    """A dense INT8 GEMM ceiling measured in the same run: torch._int_mm (cuBLASLt)
    at size^3, as back-to-back calls in one CUDA graph.  None if it does not run."""
    try:
        a = torch.randint(-127, 128, (size, size), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (size, size), dtype=torch.int8, device=dev)
        c = torch.empty(size, size, dtype=torch.int32, device=dev)
        stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(stream):
            us = _graph_us(stream, dev, lambda i: torch._int_mm(a, b, out=c), n)
        return {"tops": 2.0 * size ** 3 / (us * 1e-6) / 1e12, "us": us,
                "how": f"torch._int_mm {size}^3, {n} back-to-back calls in one CUDA graph"}
    except Exception as ex:  # a side measurement never takes the bench line down
        return {"error": str(ex)[:200]}


def secondary_workload(name, dev, steps=20):
    """A short measurement of another workload in the same run (the metric also names
    prefill M=4096): K steps of act-quant + GEMM in one CUDA graph, then K back-to-back
    GEMMs in another for the GEMM's own duration per launch."""
    import w4a8_bit_weight_b200 as lq
    from w4a8_bit_weight_b200 import synth
    w = synth.WORKLOADS[name]
    X, W = synth.make_workload(w)
    qw, s_u8, a_u8, s_c = lq.lq_quantize_weights(W.to(dev))
    wset_bytes = qw.numel() + s_u8.numel() + a_u8.numel() + 4 * s_c.numel()
    n_sets = min(64, max(4, int(np.ceil(3 * L2_BYTES / wset_bytes))))
    sets = [(qw, s_u8, a_u8, s_c)] + [(qw.clone(), s_u8.clone(), a_u8.clone(), s_c.clone())
                                      for _ in range(n_sets - 1)]
    Xd = X.to(dev)
    res = {"workload": w.note}
    stream = torch.cuda.Stream(dev)
    for M in w.Ms:
        xq = torch.empty(M, w.K, dtype=torch.int8, device=dev)
        sx = torch.empty(M, dtype=torch.float32, device=dev)
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
        cnt = [0]

        def one(quant=True):
            if quant:
                lq.lq_quantize_act(Xd[:M], out=(xq, sx))
            wq = sets[cnt[0] % n_sets]
            cnt[0] += 1
            lq.lq_w4a8_gemm(xq, sx, *wq, out=out)

        def time_graph(g):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b) / steps

        with torch.cuda.stream(stream):
            for _ in range(3):
                one()
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(steps):
                    one()
            gi = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gi, stream=stream):
                for _ in range(steps):
                    one(quant=False)
            g.replay()
            gi.replay()
            torch.cuda.synchronize(dev)
            ms = time_graph(g)
            gemm_ms = time_graph(gi)
        ops = 2.0 * M * w.N * w.K
        res[str(M)] = {"ms_per_step": ms, "tops_step": ops / (ms * 1e-3) / 1e12,
                       "gemm_us": 1e3 * gemm_ms, "gemm_tops": ops / (gemm_ms * 1e-3) / 1e12,
                       "gemm_gbs": gemm_bytes(M, w.N, w.K) / (gemm_ms * 1e-3) / 1e9}
    st = lq.lq_get_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error in the {name} measurement: {st}")
    return res


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    from w4a8_bit_weight_b200 import synth
    if rank != 0:
        return None
    w = synth.WORKLOADS[args.workload]
    steps = max(1, args.steps)
    cb = cpu_baseline(w, budget_s=min(60.0, 2.0 + 0.1 * steps))
    return {
        "metric": "W4A8 GEMM TOPS and HBM GB/s vs roofline at decode M=1-16 and prefill M=4096",
        "impl": "reference", "value": cb["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic", "config": {"workload": w.note, "M": list(w.Ms), "N": w.N, "K": w.K},
        "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            res = run_ours(args, rank, world, local_rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
