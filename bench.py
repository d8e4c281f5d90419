#!/usr/bin/env python
"""Throughput of Hessian-aware layer quantization (H + factor + GPTQ column loop) on B200.

One step = one whole layer through the C ABI: H = 2 X^T X from the calibration tokens, the
dead-feature fix / damping / factor of H_d^-1, and the GPTQ column loop with lazy updates,
packing and losses.  The default workload is the largest single-GPU layer of the recipes: the
MLP down projection W 4096 x 14336 bf16 with 8192 calibration tokens (3-bit asymmetric, group
128), whose factor is 14336 wide.  ``--workload sweep_block`` runs one block of the 8B-shaped
sweep instead (q, k, v, o, gate, up, down at 2-bit group 64, four shared Hessians): a step is
the whole block.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gq|reference] [--workload NAME]

Multi-GPU (launched by torchrun): every rank quantizes its own layer (independent problems,
no data-path collective), so the job's throughput is the sum over ranks (weak scaling); the
timed region is bracketed by barriers and its duration is the max over ranks.

Roofline: every stage is reported against the pipe it runs on, with peaks measured in this
process before the timed region (cuBLAS fp64, tf32, fp32 and int8 GEMMs; HBM and bf16 from
MEASURED_PEAKS.json), and the whole step against the sum of the stages' floors.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "weights quantized/s per linear layer (H+Cholesky+GPTQ), % of roofline, 1×B200"
UNIT = "weights/s"
DEFAULT_WORKLOAD = "mlp_down_4096x14336"
SWEEP_WORKLOAD = "sweep_block"
L2_FLUSH_BYTES = 256 << 20

# int8 digit products the Hessian kernel issues per multiply-add of X^T X (four 7-bit digits a
# value, the 13 pairs of digits with a + b <= 4)
HESSIAN_DIGIT_PRODUCTS = 13


# ---------------------------------------------------------------------------------------------
# distributed plumbing (host side; covered by gloo tests on CPU)
# ---------------------------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def dist_init(backend: str, timeout_s: float = 120.0):
    import datetime
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return ws, rank


def reduce_max(value: float, device) -> float:
    """Max of a host float over ranks (identity when not distributed)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def job_throughput(weights_per_rank: int, n_ranks: int, steps: int, max_ms: float) -> float:
    """Whole-job weights/s: every rank quantizes `steps` layers; time is the slowest rank's."""
    return weights_per_rank * n_ranks * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, local_rank: int, period_ms: int = 50):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v for v in vis.split(",") if v.strip() != ""]
        self.phys = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.phys, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = [l.strip().split(",") for l in open(self.path) if l.strip()]
        os.unlink(self.path)
        return self.summarise(rows)

    @classmethod
    def summarise(cls, rows):
        """Median SM clock and the throttle reasons seen, from nvidia-smi csv rows."""
        sm, mx, reasons = [], [], set()
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(cls.REASONS, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# roofline denominators
# ---------------------------------------------------------------------------------------------

def file_peaks():
    """HBM copy bandwidth and bf16 GEMM throughput measured on this machine (MEASURED_PEAKS.json),
    else the earlier measurement kept as the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0)}, "measured (MEASURED_PEAKS.json)"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


def _best_ms(fn, reps: int, warm: int = 2) -> float:
    for _ in range(warm):
        fn()
    best = float("inf")
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    return best


def measure_pipe_peaks(device, size: int = 8192) -> dict:
    """Throughput of the pipes this path runs on that MEASURED_PEAKS.json does not hold, each a
    cuBLAS GEMM of size^3 timed with CUDA events (best of 5 after 2 warm-ups): fp64 (the fp64
    tensor/FMA units), tf32 (tensor cores), fp32 without tf32 (the FFMA units) and int8 (tensor
    cores, int32 accumulation; ops = 2 size^3).  Compute only: no clock or power setting is
    read or changed."""
    torch.cuda.set_device(device)
    out = {}
    flops = 2.0 * size ** 3
    prec = torch.get_float32_matmul_precision()

    def gemm(dtype, mode=None, reps=5, warm=2):
        a = torch.randn(size, size, dtype=dtype, device=device)
        b = torch.randn(size, size, dtype=dtype, device=device)
        if mode:
            torch.set_float32_matmul_precision(mode)
        return flops / (_best_ms(lambda: a @ b, reps, warm) * 1e-3) / 1e12

    def int8():
        ai = torch.randint(-64, 64, (size, size), dtype=torch.int8, device=device)
        bi = torch.randint(-64, 64, (size, size), dtype=torch.int8, device=device).t()
        return flops / (_best_ms(lambda: torch._int_mm(ai, bi), 5) * 1e-3) / 1e12

    probes = {"fp64_tflops": lambda: gemm(torch.float64, reps=3, warm=1),
              "fp32_tflops": lambda: gemm(torch.float32, "highest", reps=3, warm=1),
              "tf32_tflops": lambda: gemm(torch.float32, "high"),
              "int8_tops": int8}
    for key, fn in probes.items():
        try:
            out[key] = fn()
        except Exception as e:  # recorded; the caller falls back to a nominal ratio
            out.setdefault("unmeasured", []).append(f"{key}: {type(e).__name__}")
        finally:
            torch.set_float32_matmul_precision(prec)
            torch.cuda.empty_cache()
    return out


# nominal dense ratios to the bf16 peak (B200: bf16 2.25 PF, tf32 1.1 PF, int8 4.5 POPS,
# fp64 40 TF, fp32 80 TF), used only for a pipe whose GEMM could not be measured
NOMINAL_TO_BF16 = {"fp64_tflops": 40 / 2250, "fp32_tflops": 80 / 2250,
                   "tf32_tflops": 1125 / 2250, "int8_tops": 2.0}


def complete_peaks(peaks: dict) -> dict:
    for key, ratio in NOMINAL_TO_BF16.items():
        if key not in peaks:
            peaks[key] = peaks["bf16_tflops"] * ratio
            peaks.setdefault("derived", []).append(f"{key} = bf16 x nominal ratio {ratio:.4f}")
    return peaks


# ---------------------------------------------------------------------------------------------
# the work of a step and its floor on each pipe
# ---------------------------------------------------------------------------------------------

# The factor's schedule (gq_factor.cu): from n = 1536, 512-wide super-panels; the trailing
# update of every super-panel that has rows below it (next super-panel's columns and all later
# ones: the lower triangle of the remaining (n - sp1) x (n - sp1) block, depth 512) and the
# inverse's block product T[sp1:, :sp0] += L[sp1:, K] X[K, :sp0] run as int8 digit products,
# 21 per multiply-add (six 7-bit digits a value, the pairs with p + q <= 5).
FACTOR_SUPER = 512  # the split path's super-panel width (products of depth 512)
FACTOR_SPLIT_MIN_N = 1536
FACTOR_DIGIT_PRODUCTS = 21


# DRAM bytes (read + written) of one call of a stage, from one ncu capture of every kernel of
# that call (dram__bytes_read.sum + dram__bytes_write.sum, one pass each), keyed by stage and
# width; valid only for the kernels as captured (commit 0b9f7bc).
STAGE_DRAM_BYTES = {
    ("factor", 4096): {"bytes": 1.374e9,
                       "source": "ncu dram__bytes_read.sum + dram__bytes_write.sum over the 238 "
                                 "kernels of one gq_prepare_hinv call at n = 4096 (cold caches "
                                 "between kernels; kernels of commit 0b9f7bc)"},
    ("factor", 14336): {"bytes": 4.029e10,
                        "source": "ncu dram__bytes_read.sum + dram__bytes_write.sum over the 858 "
                                  "kernels of one gq_prepare_hinv call at n = 14336 (one pass "
                                  "each, cold caches between kernels; kernels of commit "
                                  "0b9f7bc)"},
}


def stage_traffic(stage: str, layers, sweep: bool):
    """The measured DRAM traffic of one call of ``stage`` for a single-layer step whose width
    was captured, else None (a sweep step runs several widths)."""
    if sweep or len(layers) != 1:
        return None
    return STAGE_DRAM_BYTES.get((stage, layers[0][2]))


def factor_work(n: int):
    """(multiply-adds done as int8 digit products, remaining fp64 flops) of one factor of
    width n; the two add up to the algorithmic 2 n^3 / 3 flops."""
    total = 2.0 * n ** 3 / 3.0
    if n < FACTOR_SPLIT_MIN_N:
        return 0.0, total
    macs = 0.0
    K = FACTOR_SUPER
    for sp0 in range(0, n, K):
        sp1 = sp0 + K
        if sp1 > n:
            break  # a narrower last block row: its inverse products stay fp64
        r = n - sp1
        # trailing update of the rest (lower triangle) and the inverse's T[k1:, <k0] += L X
        macs += (r * (r + 1) / 2.0 + r * sp0) * K
        # the inverse's full-width block row products with the triangular X_KK (half of its
        # K x K entries are zero: the algorithmic count is half the issued one):
        # T[k1:, K] = L X_KK and X[K, <k0] = -X_KK T
        macs += (r * K * K + K * sp0 * K) / 2.0
    return macs, max(total - 2.0 * macs, 0.0)


def step_shapes(workload: str, spec: dict):
    """(inputs [(key, n, T)], layers [(name, m, n, key)]) of one step."""
    if workload == SWEEP_WORKLOAD:
        from post_weight_quantization_22_b200 import synth
        inputs, layers = [], []
        for name, m, n, key in synth.SWEEP_LAYERS:
            if key not in [i[0] for i in inputs]:
                inputs.append((key, n, synth.SWEEP_T))
            layers.append((name, m, n, key))
        return inputs, layers
    return [("x", spec["n"], spec["T"])], [("w", spec["m"], spec["n"], "x")]


def stage_model(inputs, layers, bits: int, group: int, w_bytes: int, peaks: dict,
                stage_ms: dict) -> tuple[dict, dict]:
    """Per-stage algorithmic work, the floor time on the pipe each stage runs on, and the
    achieved fraction; plus the whole step against the sum of the floors (as built) and
    against the floors of the nominal-precision plan (bf16 H, 3xTF32 factor and lazy updates,
    FP32 column recursion, HBM packing)."""
    hbm = peaks["hbm_gbs"] * 1e9
    fp64 = peaks["fp64_tflops"] * 1e12
    tf32 = peaks["tf32_tflops"] * 1e12
    fp32 = peaks["fp32_tflops"] * 1e12
    int8 = peaks["int8_tops"] * 1e12
    bf16 = peaks["bf16_tflops"] * 1e12
    h_macs = sum(n * (n + 1) / 2 * T for _, n, T in inputs)
    f_flops = sum(2.0 * n ** 3 / 3 for _, n, _ in inputs)
    f_split = [factor_work(n) for _, n, _ in inputs]
    f_int8_ops = sum(2.0 * macs * FACTOR_DIGIT_PRODUCTS for macs, _ in f_split)
    f_fp64 = sum(fp for _, fp in f_split)
    lazy_flops = sum(float(m) * n * n for _, m, n, _ in layers)
    loop_bytes = 0.0
    for _, m, n, _ in layers:
        G = 1 if group == 0 else -(-n // group)
        loop_bytes += m * n * w_bytes + n * n / 2 * 4 + m * n * bits / 8 + m * G * 5
    t = {
        "hessian": 2 * h_macs * HESSIAN_DIGIT_PRODUCTS / int8,
        "factor": f_int8_ops / int8 + f_fp64 / fp64,
        "column_loop": max(3 * lazy_flops / tf32, loop_bytes / hbm),
    }
    stages = {
        "hessian": dict(work=2 * h_macs, unit="flop", pipe="int8 tensor cores",
                        issued=f"{HESSIAN_DIGIT_PRODUCTS} int8 digit products per multiply-add",
                        peak=f"{peaks['int8_tops']:.0f} TOPS int8 (cuBLAS, measured here)"),
        "factor": dict(work=f_flops, unit="flop", pipe="int8 tensor cores + fp64 tensor cores",
                       issued=(f"{f_int8_ops / 2 / FACTOR_DIGIT_PRODUCTS / (f_flops / 2):.3f} of "
                               f"the multiply-adds as {FACTOR_DIGIT_PRODUCTS} int8 digit products "
                               f"each, the rest fp64 (DMMA m16n8k8 and DFMA)"),
                       peak=(f"{peaks['int8_tops']:.0f} TOPS int8 and {peaks['fp64_tflops']:.1f} "
                             f"TFLOP/s fp64 (cuBLAS, measured here)")),
        "column_loop": dict(work=lazy_flops, unit="flop", pipe="tf32 tensor cores / HBM",
                            issued="3xTF32 lazy updates; floor also >= algorithmic HBM bytes",
                            bytes=loop_bytes,
                            peak=f"{peaks['tf32_tflops']:.0f} TFLOP/s tf32 (cuBLAS, measured "
                                 f"here), {peaks['hbm_gbs']:.0f} GB/s HBM"),
    }
    for k, st in stages.items():
        ms = stage_ms[k]
        st["ms"] = round(ms, 4)
        st["t_roof_ms"] = round(t[k] * 1e3, 4)
        st["frac"] = round(t[k] * 1e3 / ms, 4)
        st["achieved_tflops"] = round(st["work"] / (ms * 1e-3) / 1e12, 3)
    total = sum(stage_ms.values())
    survey = (2 * h_macs / bf16 + f_flops / (tf32 / 3) + lazy_flops / (tf32 / 3)
              + sum(max(2.0 * m * n * 128 / fp32,
                        (m * n * w_bytes + n * n / 2 * 4) / hbm) for _, m, n, _ in layers)
              + sum(m * n * bits / 8 / hbm for _, m, n, _ in layers))
    overall = {"t_ms": round(total, 4),
               "t_roof_ms_as_built": round(sum(t.values()) * 1e3, 4),
               "frac_as_built": round(sum(t.values()) * 1e3 / total, 4),
               "t_roof_ms_survey": round(survey * 1e3, 4),
               "frac_survey": round(survey * 1e3 / total, 4)}
    return stages, overall


# ---------------------------------------------------------------------------------------------
# the CPU oracle as a baseline (bounded samples)
# ---------------------------------------------------------------------------------------------

def oracle_layer_sample(problems, tokens: int, n_sub: int, rows: int, seed: int = 0):
    """Time the fp64 oracle on a bounded sample of a step and scale each part to the full step
    by its operation count.  ``problems``: [(X, [(W, bits, group)...])], layers sharing X.

    Per input: H on the first ``tokens`` tokens (cost proportional to T), the factor of the
    leading n_sub x n_sub block of the damped H (cost proportional to n^3); per layer: the GPTQ
    column loop on ``rows`` sampled rows over those n_sub columns (cost proportional to m n^2).
    Returns (total seconds extrapolated, detail)."""
    from oracle import gptq_oracle as O
    rng = np.random.default_rng(seed)
    total, det = 0.0, {"hessian_s": 0.0, "factor_s": 0.0, "loop_s": 0.0, "measured_s": 0.0}
    for X, layers in problems:
        T, n = X.shape
        tk, ns = min(tokens, T), min(n_sub, n)
        t0 = time.perf_counter()
        H = O.hessian(X[:tk])
        t1 = time.perf_counter()
        hfix, _, _ = O.fix_dead_features(H[:ns, :ns], np.zeros((1, ns)))
        hd, _ = O.dampen(hfix, 0.01)
        U = O.hinv_upper_factor(hd)
        t2 = time.perf_counter()
        det["hessian_s"] += (t1 - t0) * T / tk
        det["factor_s"] += (t2 - t1) * (n / ns) ** 3
        det["measured_s"] += t2 - t0
        for W, bits, group in layers:
            m = W.shape[0]
            sel = rng.choice(m, size=min(rows, m), replace=False)
            t3 = time.perf_counter()
            O.gptq_columns(W[sel][:, :ns], U, bits, group=group)
            t4 = time.perf_counter()
            det["loop_s"] += (t4 - t3) * (m / len(sel)) * (n / ns) ** 2
            det["measured_s"] += t4 - t3
    total = det["hessian_s"] + det["factor_s"] + det["loop_s"]
    return total, det


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def workload_data(workload: str):
    """(problems for the oracle, GPU inputs, spec, weights per step).  problems:
    [(X fp64, [(W fp64, bits, group)])]."""
    from post_weight_quantization_22_b200 import synth
    if workload == SWEEP_WORKLOAD:
        Ws, Xs = synth.sweep_block(0)
        spec = dict(m=None, n=None, T=synth.SWEEP_T, bits=2, group=64, reverse=0, clip=1,
                    dtype="bf16")
        problems = []
        for key in Xs:
            lay = [(Ws[name].double().numpy(), 2, 64)
                   for name, _, _, k in synth.SWEEP_LAYERS if k == key]
            problems.append((Xs[key].double().numpy(), lay))
        weights = sum(m * n for _, m, n, _ in synth.SWEEP_LAYERS)
        return problems, (Ws, Xs), spec, weights
    W, X, spec = synth.workload(workload)
    problems = [(X.double().numpy(), [(W.double().numpy(), spec["bits"], spec["group"])])]
    return problems, (W, X), spec, spec["m"] * spec["n"]


# ---------------------------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------------------------

def run_gq(args):
    from post_weight_quantization_22_b200 import gq as G
    from post_weight_quantization_22_b200 import synth
    from post_weight_quantization_22_b200.pipeline import BlockQuantizer, LayerQuantizer

    ws, rank = dist_init("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    sweep = args.workload == SWEEP_WORKLOAD
    problems, data, spec, weights = workload_data(args.workload)
    stream = torch.cuda.current_stream(device)

    if sweep:
        Ws, Xs = data
        cfg = G.QuantCfg(bits=2, group_size=64)
        bq = BlockQuantizer(synth.SWEEP_LAYERS, cfg, device=device, max_tokens=synth.SWEEP_T)
        Wd = {k: v.to(device) for k, v in Ws.items()}
        Xd = {k: v.to(device) for k, v in Xs.items()}

        def st_hessian():
            for key in bq.inputs:
                bq.hessian(key, Xd[key])

        def st_prepare():
            for key in bq.inputs:
                bq.prepare(key)

        def st_quantize():
            for name, _, _, _ in bq.layers:
                bq.quantize(name, Wd[name])

        def check():
            st = bq.status()
            if st != 0:
                raise RuntimeError(f"device status {st}")
        w_bytes = 2
    else:
        W, X = data
        m, n, T = spec["m"], spec["n"], spec["T"]
        cfg = G.QuantCfg(bits=spec["bits"], group_size=spec["group"],
                         reverse=bool(spec["reverse"]), clip=bool(spec["clip"]))
        Wd, Xd = W.to(device), X.to(device)
        lq = LayerQuantizer(m, n, cfg, device=device, order=args.order, max_tokens=T)

        def st_hessian():
            lq.hessian(Xd)

        def st_prepare():
            lq.prepare()

        def st_quantize():
            lq.quantize(Wd)

        def check():
            st = lq.status()
            if st[0] != 0 or st[1] != 0:
                raise RuntimeError(f"device status {st}")
        w_bytes = W.element_size()

    # roofline denominators, measured before anything is timed
    peaks, peak_kind = file_peaks()
    peaks.update(measure_pipe_peaks(device))
    complete_peaks(peaks)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    for _ in range(args.warmup):
        st_hessian(); st_prepare(); st_quantize()
    torch.cuda.synchronize(device)
    check()

    # ---- device-resident timing: per step [hessian | prepare | quantize] events ----
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(device)
    torch.cuda.synchronize(device)
    launches0 = G.LIB.gq_kernel_launches()
    clocks.start()
    for k in range(args.steps):
        flush.zero_()
        e = ev[k]
        e[0].record(stream)
        st_hessian()
        e[1].record(stream)
        st_prepare()
        e[2].record(stream)
        st_quantize()
        e[3].record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    launches = G.LIB.gq_kernel_launches() - launches0
    barrier(device)
    stage_ms = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in ev])
    total_ms = float(stage_ms.sum())
    max_ms = reduce_max(total_ms, device)
    value = job_throughput(weights, ws, args.steps, max_ms)
    check()

    # ---- end to end through the public API from pinned host buffers ----
    e2e = None
    if not sweep:
        Wh, Xh = W.pin_memory(), X.pin_memory()
        out_h = {"codes": torch.empty_like(lq.codes, device="cpu").pin_memory(),
                 "scales": torch.empty_like(lq.scales, device="cpu").pin_memory(),
                 "zeros": torch.empty_like(lq.zeros, device="cpu").pin_memory(),
                 "loss": torch.empty_like(lq.loss, device="cpu").pin_memory()}
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        for _ in range(args.warmup):  # untimed: the host-input path's graphs are captured here
            lq.run_host(Wh, Xh, out=out_h)
        barrier(device)
        torch.cuda.synchronize(device)
        for k in range(args.steps):
            flush.zero_()
            a, b = e2e_ev[k]
            a.record(stream)
            lq.run_host(Wh, Xh, out=out_h)  # pinned host in, pinned host out, copies overlapped
            b.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        e2e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in e2e_ev), device)
        h2d = W.numel() * W.element_size() + X.numel() * X.element_size()
        d2h = sum(t.numel() * t.element_size() for t in out_h.values())
        e2e = {"value": job_throughput(weights, ws, args.steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    else:
        # the block from pinned host tensors: every input and weight copied in, every layer's
        # codes / grids / losses copied out, inside the timed region
        Wh = {k: v.pin_memory() for k, v in Ws.items()}
        Xh = {k: v.pin_memory() for k, v in Xs.items()}
        out_h = {name: {k: torch.empty_like(t, device="cpu").pin_memory()
                        for k, t in bq.out[name].items()} for name in bq.out}

        def block_host():
            for k in Xh:
                Xd[k].copy_(Xh[k], non_blocking=True)
            for k in Wh:
                Wd[k].copy_(Wh[k], non_blocking=True)
            st_hessian(); st_prepare(); st_quantize()
            for name in out_h:
                for k, t in out_h[name].items():
                    t.copy_(bq.out[name][k], non_blocking=True)
        for _ in range(args.warmup):
            block_host()
        barrier(device)
        torch.cuda.synchronize(device)
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        for k in range(args.steps):
            flush.zero_()
            a, b = e2e_ev[k]
            a.record(stream)
            block_host()
            b.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        e2e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in e2e_ev), device)
        h2d = (sum(t.numel() * t.element_size() for t in Wh.values())
               + sum(t.numel() * t.element_size() for t in Xh.values()))
        d2h = sum(t.numel() * t.element_size() for d in out_h.values() for t in d.values())
        e2e = {"value": job_throughput(weights, ws, args.steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    check()

    # ---- rooflines ----
    inputs, layers = step_shapes(args.workload, spec)
    mean = stage_ms.mean(axis=0)
    stage_ms_d = {"hessian": float(mean[0]), "factor": float(mean[1]),
                  "column_loop": float(mean[2])}
    stages, overall = stage_model(inputs, layers, spec["bits"], spec["group"], w_bytes, peaks,
                                  stage_ms_d)
    dname = max(stage_ms_d, key=stage_ms_d.get)
    d = stages[dname]
    roof = {"kernel": {"hessian": "gq_hessian_accumulate (hessian_tc_kernel: int8 digit "
                                  "products on tcgen05)",
                       "factor": "gq_prepare_hinv (blocked Cholesky + triangular inverse: "
                                 "split_gemm_kernel int8 digit products, fp64 leaves and panels)",
                       "column_loop": "gq_quantize_layer (colloop_kernel + lazy_tc_kernel)"}[dname],
            "bound": "tensor",
            "achieved": d["achieved_tflops"],
            "peak": round(d["work"] / (d["t_roof_ms"] * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s", "frac": d["frac"], "traffic": None,
            "peak_source": d["peak"] + "; achieved = algorithmic flops / event-timed call"}
    tb = stage_traffic(dname, layers, sweep)
    if tb is not None:
        roof["traffic"] = tb["bytes"]
        roof["traffic_source"] = tb["source"]

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        t_est, det = oracle_layer_sample(problems, tokens=args.cpu_tokens, n_sub=args.cpu_n,
                                         rows=args.cpu_rows)
        cpu = {"value": weights / t_est, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": (f"fp64 numpy oracle, {det['measured_s']:.1f} s measured: H on "
                          f"{args.cpu_tokens} tokens (scaled by T), the factor of the leading "
                          f"{args.cpu_n}-wide block (scaled by n^3), the column loop on "
                          f"{args.cpu_rows} rows of it (scaled by m n^2); extrapolated "
                          f"{t_est:.1f} s per step")}

    cfgd = {"workload": args.workload, "tokens": spec["T"], "bits": spec["bits"],
            "group": spec["group"], "reverse": spec["reverse"], "clip": spec["clip"],
            **({"order": args.order} if args.order else {}),
            "l2": "flushed between steps (256 MiB write, untimed)",
            "parallelism": f"{ws} independent problems (one per GPU)"}
    if sweep:
        cfgd["layers"] = [f"{name} {m}x{n}" for name, m, n, _ in layers]
        cfgd["shared_hessians"] = len(inputs)
        cfgd["blocks"] = "one block per step (the 32 blocks of the sweep have the same shapes)"
    else:
        cfgd.update(m=spec["m"], n=spec["n"])
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64+f32",
        "data": "synthetic (seeded decaying-spectrum activations with outlier channels; "
                "N(0,0.02^2) weights with Student-t outlier rows)",
        "config": cfgd,
        "stages": stages,
        "roofline": roof,
        "roofline_overall": overall,
        "peaks": {k: (round(v, 2) if isinstance(v, float) else v) for k, v in peaks.items()
                  if v is not None},
        "peaks_source": f"hbm_gbs, bf16: {peak_kind}; fp64, tf32, fp32, int8: cuBLAS GEMMs "
                        f"timed in this process before the timed region",
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def run_reference(args):
    """The oracle itself, timed on the host cores (rank 0 only).  Once per arm: H (all tokens)
    and the factor of every input at full size; then each step is the column loop on
    ``--ref-rows`` sampled rows of every layer at full width.  The whole-layer time is the
    once-per-arm part plus each step's loop scaled to all rows."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from oracle import gptq_oracle as O
    problems, _, spec, weights = workload_data(args.workload)
    t0 = time.perf_counter()
    factors = []
    t_once = {"hessian_s": 0.0, "factor_s": 0.0}
    for X, layers in problems:
        a = time.perf_counter()
        H = O.hessian(X)
        b = time.perf_counter()
        hfix, _, _ = O.fix_dead_features(H, np.zeros((1, H.shape[0])))
        hd, _ = O.dampen(hfix, 0.01)
        U = O.hinv_upper_factor(hd)
        c = time.perf_counter()
        t_once["hessian_s"] += b - a
        t_once["factor_s"] += c - b
        factors.append(U)
    once = time.perf_counter() - t0

    def step(seed):
        rng = np.random.default_rng(seed)
        loop_s, scaled = 0.0, 0.0
        for (X, layers), U in zip(problems, factors):
            for W, bits, group in layers:
                m = W.shape[0]
                sel = rng.choice(m, size=min(args.ref_rows, m), replace=False)
                a = time.perf_counter()
                O.gptq_columns(W[sel], U, bits, group=group)
                b = time.perf_counter()
                loop_s += b - a
                scaled += (b - a) * m / len(sel)
        return loop_s, scaled

    for k in range(args.warmup):
        step(1000 + k)
    t1 = time.perf_counter()
    runs = [step(k) for k in range(args.steps)]
    wall = time.perf_counter() - t1
    layer_s = [once_s + scaled for once_s, (_, scaled) in
               zip([t_once["hessian_s"] + t_once["factor_s"]] * len(runs), runs)]
    value = weights * len(layer_s) / sum(layer_s)
    sample = (f"fp64 numpy oracle: H and factor of every input at full size once per arm "
              f"({t_once['hessian_s']:.1f} s + {t_once['factor_s']:.1f} s), then per step the "
              f"column loop on {args.ref_rows} sampled rows of every layer at full width, "
              f"scaled to all rows")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "tokens": spec["T"], "bits": spec["bits"],
                       "group": spec["group"],
                       **({"m": spec["m"], "n": spec["n"]} if spec.get("m") else {})},
            "ms_per_step_kind": "measured: the sampled column loop actually run per step",
            "extrapolated_ms_per_layer": 1e3 * sum(layer_s) / len(layer_s),
            "once_per_arm_s": round(once, 3),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 3)}
    print(json.dumps(line), flush=True)


def run_case(args):
    """One invocation for profilers: `searches` (the SSQR and HPTQ searches on the q_proj
    layer, event-timed, one JSON line), `layer` (the q_proj recipe at --case-n, or --workload
    at its full size when --case-n is not given, two calls so a profiler can skip the first), `factor`
    (gq_prepare_hinv on a seeded SPD fp64 H of width --case-n), or `huffman` (the Huffman
    encoder on the unconstrained-lattice codes of that layer, event-timed, one JSON line with
    its HBM roofline)."""
    from post_weight_quantization_22_b200 import gq as G
    from post_weight_quantization_22_b200 import synth
    from post_weight_quantization_22_b200.pipeline import LayerQuantizer

    torch.cuda.set_device(0)
    n = args.case_n if args.case_n is not None else 2048
    if args.case == "searches":
        W, X, spec = synth.workload("q_proj_4096x4096")
        m, n = W.shape
        lq = LayerQuantizer(m, n, G.QuantCfg(bits=4), device="cuda", max_tokens=X.shape[0])
        Wd, Xd = W.cuda(), X.cuda()
        lq.hessian(Xd)
        lq.prepare()
        torch.cuda.synchronize()

        def timed(fn, reps=3):
            fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                r = fn()
            b.record()
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps, r

        out = {"case": "searches", "workload": "q_proj_4096x4096"}
        ms, r = timed(lambda: G.gq_ssqr_quantize_layer(Wd, lq.U, lq.dead, lq.delta, bits=3,
                                                         density=0.01, steps=20))
        out.update(ssqr_3bit_density_0p01_steps_20_ms=ms,
                   ssqr_status=G.gq_workspace_status(r["ws"])[0])
        ms, r = timed(lambda: G.gq_hptq_quantize_layer(Wd, lq.U, lq.dead, lq.delta, bits=4,
                                                         budget=3.125, steps=12))
        out.update(hptq_budget_3p125_steps_12_ms=ms, hptq_alpha=float(r["alpha"].item()),
                   hptq_bits_per_weight=int(r["total_bits"].item()) / (m * n),
                   hptq_status=G.gq_workspace_status(r["ws"])[0])
        ms, _ = timed(lambda: G.gq_quantize_layer(Wd, lq.U, lq.dead, lq.delta,
                                                  G.QuantCfg(bits=4, clip="unbounded")))
        out["one_unbounded_lattice_pass_ms"] = ms
        print(json.dumps(out))
    elif args.case == "layer":
        if args.case_n is None:
            W, X, spec = synth.workload(args.workload)
        else:
            W, X, spec = synth.workload("q_proj_4096x4096", m=n, n=n, T=n)
        m, n = W.shape
        cfg = G.QuantCfg(bits=spec["bits"], group_size=spec["group"])
        lq = LayerQuantizer(m, n, cfg, device="cuda", max_tokens=X.shape[0])
        Wd, Xd = W.cuda(), X.cuda()
        for _ in range(1 if args.case_n is not None else 2):
            lq.run(Wd, Xd)
        torch.cuda.synchronize()
        print("status", lq.status())
    elif args.case == "factor":
        g = torch.Generator(device="cuda").manual_seed(0)
        X = torch.randn(n + 64, n, dtype=torch.float64, device="cuda", generator=g)
        H = 2 * (X.T @ X)
        U, dead, delta, ws = G.gq_prepare_hinv(H, 0.01)
        torch.cuda.synchronize()
        print("status", G.gq_workspace_status(ws))
    else:  # huffman: encode the unconstrained-lattice codes of the q_proj recipe, timed
        W, X, spec = synth.workload("q_proj_4096x4096", m=n, n=n, T=n)
        cfg = G.QuantCfg(bits=spec["bits"], clip="unbounded")
        lq = LayerQuantizer(n, n, cfg, device="cuda")
        lq.run(W.cuda(), X.cuda())
        codes = lq.codes
        out, ln, cw, info, ws = G.gq_huffman_encode(codes)
        bufs = dict(ws=ws, out=out, lengths=ln, cw=cw, info=info)
        for _ in range(3):
            G.gq_huffman_encode(codes, **bufs)
        torch.cuda.synchronize()
        reps = 20
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            G.gq_huffman_encode(codes, **bufs)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        total_bits = int(info[2])
        # algorithmic bytes: the codes read twice (histogram, encode; the range and tile-sum
        # passes read them again but a plain encoder needs two) and the stream written once
        nbytes = 2 * 4 * codes.numel() + total_bits / 8
        peaks, kind = file_peaks()
        gbs = nbytes / (ms * 1e-3) / 1e9
        print(json.dumps({"case": "huffman", "codes": codes.numel(), "bits_per_weight":
                          total_bits / codes.numel(), "ms": ms, "achieved_gbs": gbs,
                          "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
                          "peak_kind": kind, "status": G.gq_workspace_status(ws)[0]}))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["gq", "reference"], default="gq")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="a recipe of synth.WORKLOADS, or sweep_block")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--order", choices=["act"], default=None,
                    help="process the columns in act-order (descending Hessian diagonal)")
    ap.add_argument("--cpu-tokens", type=int, default=2048)
    ap.add_argument("--cpu-n", type=int, default=6144)
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--case", choices=["layer", "factor", "huffman", "searches"], default=None,
                    help="run one untimed invocation (for profilers) and exit")
    ap.add_argument("--case-n", type=int, default=None,
                    help="size of the case (default: 2048; `layer`: --workload at full size)")
    args = ap.parse_args(argv)
    if args.case:
        return run_case(args)
    if args.workload == SWEEP_WORKLOAD and args.order:
        ap.error("--order applies to single-layer workloads")
    if args.warmup < 3 and args.impl == "gq":
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gq(args)


if __name__ == "__main__":
    main()
