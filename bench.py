#!/usr/bin/env python
"""Benchmark of the RotateAttention INT4 attention forward on B200.

One step = one pass of the hot path over the Wan2.2-shaped workload
(B=1, H=40, N=21*45*80=75,600, d=128): ra_rotate_quantize_qkv followed by
ra_int4_attention_fwd, inputs resident in HBM.  Metric: INT4 attention TOPS
= 4*N^2*d*H / time.  Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config wan|hunyuan|half|tiny|wan_flat] [--schedule]

Besides the step, the line reports: the attention call alone against the
measured INT8 tensor-core rate (roofline), the prologue against measured HBM
bandwidth, the FP16 path, the end-to-end host-buffer call, the mixed-precision
schedule (10 steps x 10 blocks, 48 % INT4; --schedule: the 10 x 40 one), and
a stress line on flat logits (every exponential computed).

--impl reference times the CPU oracle (the only reference this method has:
the paper released no kernels) on a bounded sample of the same workload.
Multi-GPU: replicas only (the path has no exchange step); each rank runs the
same workload on its own GPU and the value is the sum over ranks, timed as
the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_quantized_attention_b200 import synth  # noqa: E402
from int4_quantized_attention_b200 import schedule as sched_mod  # noqa: E402

METRIC = "INT4 attention TOPS (4*N^2*d*H/time) and fraction of B200 INT8 tensor peak"
KERNELS_PER_STEP = 5      # qk_quant, v_amax, v_quant, expand, int4_attn
# Nominal dense tensor rates: int8 (= fp8) is twice bf16/fp16 on B200.
INT8_PER_BF16 = 2.0


def profiled_traffic(cfg):
    """DRAM bytes per launch of int4_attn_kernel from the committed ncu
    summary, or None when that capture is of another kernel source or the
    workload differs from the one the summary scales to."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "int4_attn_kernel_wanH16.md")
    src = os.path.join(ROOT, "int4_quantized_attention_b200", "csrc", "ra_attn_int4.cu")
    if cfg.name != "wan" or not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.split(":")[0].strip() in ("kernel_source_sha256", "traffic_bytes_per_launch_wan40"):
            k, val = line.split(":", 1)
            fields[k.strip()] = val.strip().split()[0]
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if fields.get("kernel_source_sha256") != sha or "traffic_bytes_per_launch_wan40" not in fields:
        return None
    return int(fields["traffic_bytes_per_launch_wan40"])


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_oracle_sample(cfg, budget_s: float = 12.0, max_rows: int = 65536):
    """Time the oracle on a bounded sample: the prologue of head 0 and the
    INT4 attention of query rows of head 0, in batches until the budget."""
    from oracle import oracle as O
    O.build_oracle()
    q, k, v = synth.make_qkv(cfg, heads=1)
    t0 = time.perf_counter()
    qz = O.quantize_head(cfg, q[0, 0], k[0, 0], v[0, 0])
    t_pro = time.perf_counter() - t0
    rng = np.random.default_rng(5)
    rows_done, t_att = 0, 0.0
    while t_att < budget_s and rows_done < max_rows:
        rows = rng.choice(cfg.N, 64, replace=False).astype(np.int64)
        t0 = time.perf_counter()
        O.attention_rows(cfg, qz, rows=rows)
        t_att += time.perf_counter() - t0
        rows_done += len(rows)
    ops = 4.0 * rows_done * cfg.N * cfg.d
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return dict(value=ops / t_att / 1e12, unit="TOPS", cores=cores, kind="oracle", cpu_model=cpu_model(),
                sample=f"{cfg.name}: INT4 attention of {rows_done} query rows of head 0 "
                       f"({rows_done * cfg.N} row-key pairs, {t_att:.1f} s); head-0 prologue "
                       f"{t_pro:.2f} s not counted in the TOPS",
                seconds=t_att)


def reference_arm(args, cfg, rank):
    if rank != 0:
        return
    cb = cpu_oracle_sample(cfg, budget_s=max(3.0, min(20.0, 4.0 * args.steps)))
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int32", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d,
                       "grid": [cfg.F, cfg.Hh, cfg.W], "n_text": cfg.n_text, "split": list(cfg.split),
                       "rotation": cfg.rot},
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "cpu_model")},
            "e2e": {"value": cb["value"], "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(x: float, device) -> float:
    """The largest per-rank value (each rank's device time): the whole job
    is as slow as its slowest replica.  A no-op for one process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tops(world: int, ops_per_replica: float, ms: float) -> float:
    """Whole-job throughput: every replica does ops_per_replica in ms."""
    return world * ops_per_replica / (ms * 1e-3) / 1e12


def event_time(fn, iters, stream):
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(iters):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / iters


def measure_int8_peak(dev, stream, local):
    """Dense INT8 tensor-core rate on this GPU, measured now: the library's
    tcgen05 kind::i8 issue loop (one CTA per SM, the attention kernel's
    operand layout), as ~50 ms launches (burst, like the attention call) and
    back to back for about a second (sustained); and cuBLASLt's int8 GEMM
    (torch._int_mm, 8192^3) for comparison."""
    import torch
    from int4_quantized_attention_b200 import api
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    ws = torch.zeros((256,), dtype=torch.uint8, device=dev)
    out = {"sms": n_sm}
    with ClockSampler(local) as clk:
        for n in (128, 256):
            ops_per_iter = n_sm * 4 * 2 * 128 * n * 32
            api.measure_mma_i8(n, 2000, n_sm, ws)          # warm-up
            t = event_time(lambda: api.measure_mma_i8(n, 20000, n_sm, ws), 1, stream)
            iters = max(1000, int(20000 * 50.0 / max(t, 1e-3)))   # ~50 ms per launch
            burst = [event_time(lambda: api.measure_mma_i8(n, iters, n_sm, ws), 1, stream) for _ in range(5)]
            ms_b = statistics.median(burst)
            reps = max(1, int(1000.0 / ms_b))
            ms_s = event_time(lambda: api.measure_mma_i8(n, iters, n_sm, ws), reps, stream)
            out[f"tcgen05_i8_n{n}"] = {"burst_tops": ops_per_iter * iters / (ms_b * 1e-3) / 1e12,
                                       "sustained_tops": ops_per_iter * iters / (ms_s * 1e-3) / 1e12,
                                       "launch_ms": ms_b, "sustained_s": reps * ms_s / 1e3}
        api.check_device_error(ws)
        try:
            m = 8192
            a = torch.randint(-8, 8, (m, m), dtype=torch.int8, device=dev)
            b = torch.randint(-8, 8, (m, m), dtype=torch.int8, device=dev).t()   # column-major
            for _ in range(3):
                torch._int_mm(a, b)
            ms1 = statistics.median([event_time(lambda: torch._int_mm(a, b), 1, stream) for _ in range(20)])
            reps = max(1, int(1000.0 / ms1))
            ms2 = event_time(lambda: torch._int_mm(a, b), reps, stream)
            out["cublaslt_int8_gemm"] = {"shape": [m, m, m], "burst_tops": 2.0 * m ** 3 / (ms1 * 1e-3) / 1e12,
                                         "sustained_tops": 2.0 * m ** 3 / (ms2 * 1e-3) / 1e12}
            del a, b
        except Exception as e:   # report, do not fail the bench
            out["cublaslt_int8_gemm"] = {"unavailable": str(e).splitlines()[0][:160]}
    out["clocks"] = clk.summary()
    best = max(out["tcgen05_i8_n128"]["burst_tops"], out["tcgen05_i8_n256"]["burst_tops"])
    best_s = max(out["tcgen05_i8_n128"]["sustained_tops"], out["tcgen05_i8_n256"]["sustained_tops"])
    out["peak_burst_tops"], out["peak_sustained_tops"] = best, best_s
    return out


def stress_flat(dev, stream, peak, heads=8, steps=5):
    """Attention call on flat logits (every P code non-zero, no exponential
    skipped): the Wan shapes with Q/K channels scaled by 0.3, on `heads` heads
    (heads are independent CTAs, so the rate per call is that of 40)."""
    import torch
    from int4_quantized_attention_b200 import api
    cfg = synth.CONFIGS["wan_flat"].replace(H=heads, name=f"wan_flat-H{heads}")
    q, k, v = (torch.from_numpy(t).to(dev) for t in synth.make_qkv(cfg))
    ra = api.RotateAttention(cfg, dev, fp16_path=False)
    out = torch.empty_like(q)
    ra.rotate_quantize(q, k, v)
    for _ in range(3):
        ra.int4_attention(out)
    ms = event_time(lambda: ra.int4_attention(out), steps, stream)
    ra.check()
    tops = cfg.ops / (ms * 1e-3) / 1e12
    return {"workload": cfg.name, "H": heads, "N": cfg.N, "int4_attention_ms": ms, "tops": tops,
            "frac_int8_peak": tops / peak}


def our_arm(args, cfg, rank, world):
    import torch
    import torch.distributed as dist
    from int4_quantized_attention_b200 import api, build

    build.build()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()

    q, k, v = synth.make_qkv(cfg)
    qd, kd, vd = (torch.from_numpy(t).to(dev) for t in (q, k, v))
    ra = api.RotateAttention(cfg, dev, fp16_path=True)
    out = torch.empty_like(qd)

    def step():
        ra.rotate_quantize(qd, kd, vd)
        ra.int4_attention(out)

    if args.only_fp16:   # the FP16 path alone (profiler captures)
        for _ in range(args.warmup):
            ra.fp16_attention(qd, kd, vd, out)
        ms = event_time(lambda: ra.fp16_attention(qd, kd, vd, out), args.steps, stream)
        ra.check()
        if rank == 0:
            print(json.dumps({"workload": cfg.name, "fp16_path_ms": ms}), flush=True)
        return
    for _ in range(args.warmup):
        step()
    ra.check()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms_step = event_time(step, args.steps, stream)
        # the dominant kernel alone, on the same stream (inputs > L2 between launches)
        ms_attn = event_time(lambda: ra.int4_attention(out), args.steps, stream)
        ms_pro = event_time(lambda: ra.rotate_quantize(qd, kd, vd), max(args.steps, 10), stream)
    ra.check()
    torch.cuda.synchronize()
    if args.only_step:
        if rank == 0:
            print(json.dumps({"workload": cfg.name, "ms_per_step": ms_step, "int4_attention_ms": ms_attn,
                              "prologue_ms": ms_pro}), flush=True)
        return
    ms_step = max_over_ranks(ms_step, dev)
    if world > 1:
        dist.barrier()

    # FP16 path on the same workload (a few calls)
    ms_f16 = event_time(lambda: ra.fp16_attention(qd, kd, vd, out), max(2, args.steps // 3), stream)
    ra.check()

    # end to end with host buffers: ra_int4_attention_host pipelines the copies
    # over chunks of heads on the copy engines while the kernels run
    qh, kh, vh = (torch.from_numpy(t).pin_memory() for t in (q, k, v))
    oh = torch.empty(out.shape, dtype=torch.float16).pin_memory()

    def e2e_step():
        ra.forward_host(qh, kh, vh, oh, heads_per_chunk=args.chunk_heads)

    def e2e_serial():
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        step()
        oh.copy_(out, non_blocking=True)

    e2e_step()
    ms_e2e = event_time(e2e_step, max(2, args.steps // 2), stream)
    ms_e2e_serial = event_time(e2e_serial, 2, stream)
    ra.check()
    ms_e2e = max_over_ranks(ms_e2e, dev)

    sched = run_schedule(ra, qd, kd, vd, out, stream,
                         sched_mod.BENCH_SCHEDULE if args.schedule else sched_mod.BENCH_SCHEDULE_SHORT)
    peak8 = measure_int8_peak(dev, stream, local)
    stress = None if args.no_stress else stress_flat(dev, stream, peak8["peak_burst_tops"])

    if rank != 0:
        return
    ops = cfg.ops
    tops = aggregate_tops(world, ops, ms_step)
    attn_tops = ops / (ms_attn * 1e-3) / 1e12
    # the attention kernel is timed alone: the burst figure of the INT8 rate probe
    peak_int8 = peak8["peak_burst_tops"]
    Np = ra.N_pad
    BH = cfg.B * cfg.H
    pro_bytes = (3 * BH * cfg.N * cfg.d * 2            # read q, k, v
                 + BH * cfg.N * cfg.d * 2              # second read of v (after its amax)
                 + 3 * BH * Np * cfg.d // 2            # packed INT4 writes
                 + BH * (Np // 64) * cfg.d * 4)        # V column sums
    cpu = cpu_oracle_sample(cfg, budget_s=12.0) if not args.no_cpu_baseline else None
    line = {
        "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8xs8->s32 (INT4 codes), fp32 softmax", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d,
                   "grid": [cfg.F, cfg.Hh, cfg.W], "n_text": cfg.n_text, "split": list(cfg.split),
                   "rotation": cfg.rot, "p_mode": cfg.p_mode, "v_rot": cfg.v_rot,
                   "parallelism": "replicas" if world > 1 else "single-gpu",
                   "l2": "inputs larger than L2 (q,k,v 2.3 GB; INT8 K/V operand images 0.77 GB per pass)"},
        "roofline": {"kernel": "int4_attn_kernel", "bound": "tensor", "achieved": attn_tops,
                     "peak": peak_int8, "unit": "TOPS", "frac": attn_tops / peak_int8, "traffic": profiled_traffic(cfg),
                     "peak_source": "measured int8: tcgen05 kind::i8 M128xNxK32 issue loop, one CTA per SM, "
                                    "~50 ms launches (burst), best of N=128/256, this run",
                     "frac_of_sustained_int8": attn_tops / peak8["peak_sustained_tops"],
                     "frac_of_bf16_derived": attn_tops / (peaks["bf16"] * INT8_PER_BF16),
                     "frac_of_nominal_4500": attn_tops / 4500.0,
                     "algorithmic_ops_per_launch": ops},
        "int8_peak": peak8,
        "int4_attention_ms": ms_attn,
        "prologue": {"ms": ms_pro, "algorithmic_bytes": pro_bytes,
                     "achieved_gbs": pro_bytes / (ms_pro * 1e-3) / 1e9,
                     "frac_hbm": pro_bytes / (ms_pro * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "fp16_path": {"ms": ms_f16, "tflops": ops / (ms_f16 * 1e-3) / 1e12,
                      "frac_bf16_peak": ops / (ms_f16 * 1e-3) / 1e12 / peaks["bf16"],
                      "frac_bf16_peak_sustained": ops / (ms_f16 * 1e-3) / 1e12 / peaks["bf16_sus"],
                      "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16']} TF/s (the call is timed alone)",
                      "int4_step_speedup": ms_f16 / ms_step},
        "e2e": {"value": aggregate_tops(world, ops, ms_e2e), "unit": "TOPS", "ms_per_step": ms_e2e,
                "h2d_bytes_per_step": 3 * BH * cfg.N * cfg.d * 2, "d2h_bytes_per_step": BH * cfg.N * cfg.d * 2,
                "api": "ra_int4_attention_host (pinned host q, k, v, o; copies overlapped over head chunks)",
                "chunks": (f"{args.chunk_heads} heads each" if args.chunk_heads else
                           f"library default: ramp 1, 1, 2, 2, ... up to {-(-BH // 8)} heads and back down, three "
                           f"staging slots"),
                "serial_ms_per_step": ms_e2e_serial},
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": None if cpu is None else {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample",
                                                                       "cpu_model")},
        "gpu": torch.cuda.get_device_name(dev),
    }
    line["schedule"] = sched
    if stress is not None:
        line["stress_flat_logits"] = stress
    print(json.dumps(line), flush=True)


def run_schedule(ra, qd, kd, vd, out, stream, schedule):
    """Mixed-precision schedule: per (step, block) the FP16 or the INT4 path,
    each call timed with events; compared with the same calls all on FP16."""
    kinds, ms = sched_mod.run(ra, qd, kd, vd, out, schedule, stream)
    per = {"int4": [t for kd_, t in zip(kinds, ms) if kd_ == "int4"],
           "fp16": [t for kd_, t in zip(kinds, ms) if kd_ == "fp16"]}
    all16 = sched_mod.Schedule(schedule.steps, schedule.blocks, schedule.steps, 0, 0, 0)
    _, ms16 = sched_mod.run(ra, qd, kd, vd, out, all16, stream)
    ra.check()
    mixed = sum(ms)
    return {"schedule": f"{schedule.steps} steps x {schedule.blocks} blocks, FP16 on the first/last "
                        f"{schedule.first_steps}/{schedule.last_steps} steps and first/last "
                        f"{schedule.first_blocks}/{schedule.last_blocks} blocks",
            "calls": len(kinds), "int4_fraction": schedule.int4_fraction,
            "int4_ms_per_call": statistics.median(per["int4"]), "fp16_ms_per_call": statistics.median(per["fp16"]),
            "mixed_total_ms": mixed, "all_fp16_total_ms": sum(ms16), "speedup_vs_all_fp16": sum(ms16) / mixed}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="wan", choices=sorted(synth.CONFIGS))
    ap.add_argument("--schedule", action="store_true",
                    help="run the 400-call mixed schedule (10 steps x 40 blocks) instead of the 100-call one")
    ap.add_argument("--no-stress", action="store_true", help="skip the flat-logit stress line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override H (smaller profiling cases)")
    ap.add_argument("--rot", default=None, choices=["none", "interleaved", "half", "full"],
                    help="override the workload's rotation mode")
    ap.add_argument("--v-rot", action="store_true", help="Hadamard on V inside the INT4 path (undone on O)")
    ap.add_argument("--p-mode", default="range", choices=["range", "symmetric"],
                    help="P quantisation of the INT4 path (range-optimised: the method)")
    ap.add_argument("--chunk-heads", type=int, default=0,
                    help="heads per chunk of the host-buffer pipeline (0: the library's default, B*H/8)")
    ap.add_argument("--only-fp16", action="store_true",
                    help="run only warm-up and timed calls of the FP16 path (for profiler captures)")
    ap.add_argument("--only-step", action="store_true",
                    help="run only the warm-up and timed INT4 steps (for profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    cfg = synth.CONFIGS[args.config]
    if args.heads:
        cfg = cfg.replace(H=args.heads, name=f"{cfg.name}-H{args.heads}")
    if args.rot is not None and args.rot != cfg.rot:
        cfg = cfg.replace(rot=args.rot, name=f"{cfg.name}-r{args.rot}")
    if args.v_rot:
        cfg = cfg.replace(v_rot=1, name=f"{cfg.name}-vrot")
    if args.p_mode != "range":
        cfg = cfg.replace(p_mode=args.p_mode, name=f"{cfg.name}-p{args.p_mode}")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, cfg, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        our_arm(args, cfg, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
