#!/usr/bin/env python
"""Throughput of Hessian-aware layer quantization (H + factor + GPTQ column loop) on B200.

One step = one whole layer through the C ABI: H = 2 X^T X from the calibration tokens, the
dead-feature fix / damping / factor of H_d^-1, and the GPTQ column loop with lazy updates,
packing and losses.  The default workload is the q_proj-shaped layer (W 4096 x 4096 bf16,
4096 calibration tokens, 4-bit asymmetric, group 128) with seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gq|reference]

Multi-GPU (launched by torchrun): every rank quantizes its own layer (independent problems,
no data-path collective), so the job's throughput is the sum over ranks (weak scaling); the
timed region is bracketed by barriers and its duration is the max over ranks.
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
DEFAULT_WORKLOAD = "q_proj_4096x4096"
L2_FLUSH_BYTES = 256 << 20


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

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v for v in vis.split(",") if v.strip() != ""]
        self.phys = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.phys, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
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
        sm, mx, reasons = [], [], set()
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(self.REASONS, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# roofline denominators
# ---------------------------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


def fp64_peak_tflops(sm_mhz: float) -> float:
    """fp64 FMA peak: 148 SMs x 64 fp64 FMA lanes x 2 flops x clock."""
    return 148 * 64 * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------------------------------------
# the CPU oracle as a baseline (bounded sample)
# ---------------------------------------------------------------------------------------------

def oracle_sample(W, X, spec, rows: int, seed: int = 0):
    """Time the fp64 oracle on the full H and factor plus the column loop of `rows` sampled
    rows, and extrapolate the loop to all rows: weights/s for the whole layer."""
    from oracle import gptq_oracle as O
    m, n = spec["m"], spec["n"]
    sel = np.random.default_rng(seed).choice(m, size=min(rows, m), replace=False)
    t0 = time.perf_counter()
    H = O.hessian(X)
    t1 = time.perf_counter()
    h_fix, w0, _ = O.fix_dead_features(H, W)
    hd, _ = O.dampen(h_fix, 0.01)
    if spec["reverse"]:
        L = np.linalg.cholesky(hd)
    else:
        U = O.hinv_upper_factor(hd)
    t2 = time.perf_counter()
    if spec["reverse"]:
        O.babai_sic_reverse(w0[sel], L, spec["bits"], clip=bool(spec["clip"]))
    else:
        O.gptq_columns(w0[sel], U, spec["bits"], group=spec["group"], clip=bool(spec["clip"]))
    t3 = time.perf_counter()
    total = (t1 - t0) + (t2 - t1) + (t3 - t2) * m / len(sel)
    return m * n / total, dict(t_hessian=t1 - t0, t_factor=t2 - t1, t_rows=t3 - t2, rows=len(sel))


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------------------------

def run_gq(args):
    from post_weight_quantization_22_b200 import gq as G
    from post_weight_quantization_22_b200 import synth
    from post_weight_quantization_22_b200.pipeline import LayerQuantizer

    ws, rank = dist_init("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    W, X, spec = synth.workload(args.workload)
    m, n, T = spec["m"], spec["n"], spec["T"]
    cfg = G.QuantCfg(bits=spec["bits"], group_size=spec["group"], reverse=bool(spec["reverse"]),
                     clip=bool(spec["clip"]))
    Wd, Xd = W.to(device), X.to(device)
    Wh, Xh = W.pin_memory(), X.pin_memory()
    lq = LayerQuantizer(m, n, cfg, device=device, order=args.order)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    # warm-up
    for _ in range(args.warmup):
        lq.run(Wd, Xd)
    torch.cuda.synchronize(device)
    st = lq.status()
    if st[0] != 0 or st[1] != 0:
        raise RuntimeError(f"device status {st}")

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
        lq.hessian(Xd)
        e[1].record(stream)
        lq.prepare()
        e[2].record(stream)
        lq.quantize(Wd)
        e[3].record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    launches = G.LIB.gq_kernel_launches() - launches0
    barrier(device)
    stage_ms = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in ev])
    total_ms = float(stage_ms.sum())
    max_ms = reduce_max(total_ms, device)
    value = job_throughput(m * n, ws, args.steps, max_ms)
    st = lq.status()
    if st[0] != 0 or st[1] != 0:
        raise RuntimeError(f"device status {st}")

    # ---- end to end through the public API from pinned host buffers ----
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

    # ---- roofline of the dominant stage ----
    peaks, peak_kind = measured_peaks()
    mean_stage = stage_ms.mean(axis=0)
    names = ["hessian", "factor", "column_loop"]
    sm_mhz = (clk or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    fp64_tf = fp64_peak_tflops(peaks.get("sm_max_mhz", 1965.0))
    work = {  # algorithmic flops per call
        "hessian": float(n) * n * T,                              # n(n+1)/2 entries x T FMAs x 2
        "factor": 2.0 * n ** 3 / 3.0,                             # Cholesky + triangular inverse
        "column_loop": float(m) * n * n,                           # in-block + lazy updates
    }
    dom = int(np.argmax(mean_stage))
    dname = names[dom]
    achieved = work[dname] / (mean_stage[dom] / 1e3) / 1e12
    roof = {"kernel": {"hessian": "hessian_tc_kernel (H += 2 X^T X, int8 digit products)",
                       "factor": "blocked fp64 Cholesky + triangular inverse",
                       "column_loop": "colloop + lazy_update"}[dname],
            "bound": "alu", "achieved": round(achieved, 3), "peak": round(fp64_tf, 2),
            "unit": "TFLOP/s", "frac": round(achieved / fp64_tf, 4),
            "peak_source": f"fp64 FMA units x max clock (148 SMs x 64 x 2 x {peaks.get('sm_max_mhz', 1965.0):.0f} MHz)",
            "traffic": None}
    stages = {nm: {"ms": round(float(mean_stage[i]), 4),
                   "tflops": round(work[nm] / (mean_stage[i] / 1e3) / 1e12, 3)}
              for i, nm in enumerate(names)}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, info = oracle_sample(W, X, spec, rows=args.cpu_rows)
        cpu = {"value": v, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": (f"fp64 numpy oracle: full H ({info['t_hessian']:.2f}s) and factor "
                          f"({info['t_factor']:.2f}s), column loop on {info['rows']} of {m} rows "
                          f"({info['t_rows']:.2f}s) extrapolated to all rows")}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64+f32",
        "data": "synthetic (seeded decaying-spectrum activations with outlier channels; "
                "N(0,0.02^2) weights with Student-t outlier rows)",
        "config": {"workload": args.workload, "m": m, "n": n, "tokens": T, "bits": spec["bits"],
                   "group": spec["group"], "reverse": spec["reverse"], "clip": spec["clip"],
                   **({"order": args.order} if args.order else {}),
                   "l2": "flushed between steps (256 MiB write, untimed)",
                   "parallelism": f"{ws} independent layers (one per GPU)"},
        "stages": stages,
        "roofline": roof,
        "roofline_peak_kind": "derived: fp64 unit counts x measured max SM clock",
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(m * n, ws, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def run_reference(args):
    """The oracle itself, timed on the host cores (rank 0 only)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from post_weight_quantization_22_b200 import synth
    W, X, spec = synth.workload(args.workload)
    Wn, Xn = W.double().numpy(), X.double().numpy()
    for _ in range(args.warmup):
        oracle_sample(Wn, Xn, spec, rows=args.ref_rows)
    vals, infos = [], []
    t0 = time.perf_counter()
    for k in range(args.steps):
        v, info = oracle_sample(Wn, Xn, spec, rows=args.ref_rows, seed=k)
        vals.append(v)
        infos.append(info)
    wall = time.perf_counter() - t0
    # whole-job value: total weights over the summed extrapolated step times
    m, n = spec["m"], spec["n"]
    step_s = [m * n / v for v in vals]
    value = m * n * args.steps / sum(step_s)
    sample = (f"fp64 numpy oracle per step: full H and factor, column loop on {args.ref_rows} "
              f"of {m} rows extrapolated to all rows")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(step_s) / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "m": m, "n": n, "tokens": spec["T"],
                       "bits": spec["bits"], "group": spec["group"]},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": wall}
    print(json.dumps(line), flush=True)


def run_case(args):
    """One invocation for profilers: `layer` (the q_proj recipe at --case-n), `factor`
    (gq_prepare_hinv on a seeded SPD fp64 H of width --case-n), or `huffman` (the Huffman
    encoder on the unconstrained-lattice codes of that layer, event-timed, one JSON line with
    its HBM roofline)."""
    from post_weight_quantization_22_b200 import gq as G
    from post_weight_quantization_22_b200 import synth
    from post_weight_quantization_22_b200.pipeline import LayerQuantizer

    torch.cuda.set_device(0)
    n = args.case_n
    if args.case == "layer":
        W, X, spec = synth.workload(DEFAULT_WORKLOAD, m=n, n=n, T=n)
        cfg = G.QuantCfg(bits=spec["bits"], group_size=spec["group"])
        lq = LayerQuantizer(n, n, cfg, device="cuda")
        lq.run(W.cuda(), X.cuda())
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
        W, X, spec = synth.workload(DEFAULT_WORKLOAD, m=n, n=n, T=n)
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
        peaks, kind = measured_peaks()
        gbs = nbytes / (ms * 1e-3) / 1e9
        print(json.dumps({"case": "huffman", "codes": codes.numel(), "bits_per_weight":
                          total_bits / codes.numel(), "ms": ms, "achieved_gbs": gbs,
                          "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
                          "peak_kind": kind, "status": G.gq_workspace_status(ws)[0]}))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["gq", "reference"], default="gq")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--order", choices=["act"], default=None,
                    help="process the columns in act-order (descending Hessian diagonal)")
    ap.add_argument("--cpu-rows", type=int, default=256)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--case", choices=["layer", "factor", "huffman"], default=None,
                    help="run one untimed invocation (for profilers) and exit")
    ap.add_argument("--case-n", type=int, default=2048)
    args = ap.parse_args(argv)
    if args.case:
        return run_case(args)
    if args.warmup < 3 and args.impl == "gq":
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gq(args)


if __name__ == "__main__":
    main()
