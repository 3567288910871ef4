#!/usr/bin/env python
"""Benchmark of the BinaryAttention forward pass (one step = one ba_attention_fwd call:
sign pack + mu, V quantiser, fused binary-QK / int8-PV attention) on synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sweep32768_d128|deit_b|tiny|dit256|dit512|dit1024|sweep<N>_d<d>]

The default workload is the largest single-GPU configuration of the long-sequence sweep
(B=1, H=16, N=32768, d=128, bf16, 2-D relative-position bias on a 128 x 256 grid); the
others are there for measurement of the smaller shapes. Prints ONE JSON line on rank 0.
Under torchrun (N > 1) every rank runs the same workload on its own GPU (independent
replicas: the path has no data-path exchange) and the time is the max over ranks.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BinaryAttention fwd effective TOPS & tokens/s at 1 B200; % of int8 tensor peak"
UNIT = "TOPS"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
STAGES = ["stream_qkv", "finalize", "quant_v", "attention"]
KERNEL_FILES = {"stream_qkv": "prep.cu", "finalize": "prep.cu", "quant_v": "prep.cu",
                "attention_simt": "attn_simt.cu", "attention_tcgen05": "attn_tc.cu"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0 = about one second of work)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="sweep32768_d128")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (small profiling cases)")
    ap.add_argument("--attn-impl", choices=["auto", "simt", "tcgen05"], default="auto")
    ap.add_argument("--rotate", type=int, default=0, help="input sets cycled to defeat L2 (0 = auto)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def file_hash(name):
    with open(os.path.join(ROOT, "bit_qk_attention_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, only while the kernel's source is
    unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(f"{kernel}|{workload}")
    if not e or e.get("source_sha") != file_hash(KERNEL_FILES[kernel]):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def max_over_ranks(ms: float, dist, device) -> float:
    """The job's time: the largest of the ranks' device times (all ranks take part)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ops: float, tokens: float, ms_per_step: float, world: int):
    """Whole-job effective TOPS and tokens/s: every rank runs the same step on its own replica
    of the workload (weak scaling), so the job does world times the work in the slowest rank's
    time."""
    sec = ms_per_step / 1e3
    return world * ops / sec / 1e12, world * tokens / sec


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def work_units(w):
    ops = 4.0 * w.B * w.H * w.N * w.N * w.d
    return ops, w.B * w.N


def workload_config(w):
    """The workload both arms report on: shape, dtype, bias form and the key-block size of the
    quantisation contract (128 keys, the definition's block)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "io_dtype": w.dtype_name,
            "bias": {0: "none", 1: "dense", 2: "relpos2d"}[w.bias_kind], "kv_block": 128}


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(w, budget_s: float, threads: int):
    """Times the oracle on a bounded sample of the workload: whole (b,h) slices for short
    sequences, sampled query rows of one batch for long ones. Returns (ops, seconds, desc)."""
    import numpy as np
    import oracle
    o = oracle.get()
    q, k, v = w.q[:1].float().numpy(), w.k[:1].float().numpy(), w.v[:1].float().numpy()
    b1 = oracle.Bias()
    if w.bias_kind != 0:
        data = w.bias[:1] if (w.bias_kind == 1 and w.batch_stride) else w.bias
        b1 = oracle.Bias(w.bias_kind, data.float().numpy(), w.batch_stride, w.grid_h, w.grid_w, w.table_h,
                         w.table_w, w.n_prefix)
    # calibrate on a few rows of batch 0, then size the sample to the budget
    rows = np.arange(min(w.N, 8), dtype=np.int64)
    t0 = time.perf_counter()
    o.attention_fwd(q, k, v, b1, rows=rows, num_threads=threads)
    t_cal = max(time.perf_counter() - t0, 1e-4)
    per_row = t_cal / (len(rows) * w.H)
    total_rows = max(1, int(budget_s / (per_row * w.H)))
    if total_rows >= w.N:  # whole (b, h) slices of the first nb batches
        nb = int(min(w.B, total_rows // w.N))
        q, k, v = w.q[:nb].float().numpy(), w.k[:nb].float().numpy(), w.v[:nb].float().numpy()
        if w.bias_kind == 1 and w.batch_stride:
            b1.data = w.bias[:nb].float().numpy()
        rows, nr = None, w.N
    else:  # evenly spaced query rows of batch 0 (all keys)
        nb, nr = 1, total_rows
        rows = np.linspace(0, w.N - 1, nr).astype(np.int64)
    t0 = time.perf_counter()
    o.attention_fwd(q, k, v, b1, rows=rows, num_threads=threads)
    dt = time.perf_counter() - t0
    ops = 4.0 * nb * w.H * nr * w.N * w.d
    desc = (f"{nb} of {w.B} batches x {w.H} heads, {nr} of {w.N} query rows against all {w.N} keys, "
            f"{threads} threads")
    if nb < w.B or nr < w.N:
        desc += ("; extrapolated: the rate over these rows stands for the whole workload (rows are "
                 "independent and cost the same)")
    return ops, dt, desc


def run_reference(args):
    world, rank, _ = dist_info()
    if rank != 0:
        return 0
    from bit_qk_attention_b200 import inputs
    w = inputs.by_name(args.workload)
    threads = os.cpu_count() or 1
    per_step = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, per_step, threads)
    tot_ops, tot_s, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        ops, dt, desc = oracle_sample(w, per_step, threads)
        tot_ops += ops
        tot_s += dt
    value = tot_ops / tot_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64+f32",
            "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist
    world, rank, local = dist_info()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    import bit_qk_attention_b200 as ba
    from bit_qk_attention_b200 import build, inputs
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        dist.barrier()
    ba.lib()
    ba.set_attention_impl({"auto": 0, "simt": 1, "tcgen05": 2}[args.attn_impl])

    w = inputs.by_name(args.workload)
    if args.batch:
        w.B = args.batch
        w.q, w.k, w.v = (t[:args.batch].contiguous() for t in (w.q, w.k, w.v))
        w.name = f"{w.name}[B={args.batch}]"
    ops, tokens = work_units(w)
    E = w.B * w.H * w.N * w.d
    esz = 2
    set_bytes = 4 * E * esz + ba.workspace_bytes(w.B, w.H, w.N, w.d)
    R = args.rotate or max(1, min(8, -(-512 * 2 ** 20 // set_bytes)))  # cycle >= 512 MB (> 126 MB L2)
    qs = [w.q.to(dev) for _ in range(R)]
    ks = [w.k.to(dev) for _ in range(R)]
    vs = [w.v.to(dev) for _ in range(R)]
    outs = [torch.empty_like(qs[0]) for _ in range(R)]
    wss = [torch.empty(ba.workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev) for _ in range(R)]
    bias = ba.bias_from_workload(w, dev)
    stream = torch.cuda.current_stream()

    def step(i):
        j = i % R
        ba.attention_fwd(qs[j], ks[j], vs[j], bias, out=outs[j], workspace=wss[j])

    w0 = torch.cuda.Event(enable_timing=True)
    w1 = torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for i in range(args.warmup):
        step(i)
    w1.record(stream)
    torch.cuda.synchronize()
    impl_used = {1: "simt", 2: "tcgen05"}.get(ba.last_attention_impl(), "?")
    if args.steps <= 0:  # about one second of timed work, the same count on every rank
        per = w0.elapsed_time(w1) / max(1, args.warmup)
        steps = max(20, min(20000, int(1000.0 / max(per, 1e-3))))
        if world > 1:
            t = torch.tensor([steps], dtype=torch.int64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MIN)
            steps = int(t.item())
        args.steps = steps

    clocks = ClockSampler(dev.index)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    ms_per_step = ms / args.steps
    value, tok_s = job_throughput(ops, tokens, ms_per_step, world)
    ba.check_device_status()

    # Per-stage device times (a separate pass with CUDA events around each kernel).
    nst = min(args.steps, 400)
    ba.stage_timing(True)
    for i in range(nst):
        step(i)
    torch.cuda.synchronize()
    stage_ms, ncalls = ba.stage_times()
    ba.stage_timing(False)
    stage_avg = [x / max(1, ncalls) for x in stage_ms]

    peaks = load_peaks()
    int8_tops = 2.0 * peaks["bf16_tflops"]  # nominal int8:bf16 ratio of 2 on B200
    hbm = peaks["hbm_gbs"]
    dp = ba.v_row_bytes(w.d)
    BH, N, d = w.B * w.H, w.N, w.d
    nchunk = -(-N // 128)
    bias_bytes = 0 if w.bias is None else w.bias.numel() * 4
    if ba.prep_fused(w.B, w.H, N, d):
        # one launch: q, k, v read once from HBM (v's second pass hits L2), sign rows, int8 V
        # rows, mu and the V scales written; the finalize and quantise stages are empty
        prep_bytes = {"stream_qkv": 3 * E * esz + 2 * BH * N * 16 + BH * N * dp + BH * 4 * (d + 2),
                      "finalize": 0, "quant_v": 0}
    else:
        # two launches: the streaming kernel reads q, k, v and writes sign rows, per-chunk |x| sums
        # and per-group V channel maxima; the quantiser reads V again (the scales need the whole
        # slice's maxima first) and the partials, and writes int8 V, the scales and mu
        nparts = -(-nchunk // 8) if d % 8 == 0 else nchunk
        partials = 2 * BH * nchunk * 8 + BH * nparts * dp * 4
        prep_bytes = {"stream_qkv": 3 * E * esz + 2 * BH * N * 16 + partials,
                      "finalize": 0,
                      "quant_v": E * esz + partials + BH * N * dp + BH * 4 * (d + 2)}
    alg_bytes = {
        **prep_bytes,
        "attention": 2 * BH * N * 16 + BH * N * dp + E * esz + bias_bytes + BH * 4 * (d + 2),
    }
    dom = max(range(4), key=lambda k: stage_avg[k])
    name = STAGES[dom]
    t_dom = stage_avg[dom] / 1e3
    kernel = name if name != "attention" else f"attention_{impl_used}"
    if name == "attention" and ops / (int8_tops * 1e12) > alg_bytes[name] / (hbm * 1e9):
        achieved = ops / t_dom / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": int8_tops, "unit": "TOPS",
                "frac": achieved / int8_tops}
    else:
        achieved = alg_bytes[name] / t_dom / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm}
    roof.update({"kernel": kernel, "traffic": recorded_traffic(kernel, w.name),
                 "algorithmic_bytes": alg_bytes[name], "launch_ms": stage_avg[dom],
                 "peak_source": f"{peaks['source']} ({'int8 = 2 x bf16 burst' if roof['bound'] == 'tensor' else 'copy burst'})"})
    attn_ms = stage_avg[3]
    # The preparation kernels against HBM (stages with no work, as on the one-launch path,
    # are left out).
    prep_stages = [k for k in range(3) if alg_bytes[STAGES[k]] > 0]
    prep_t = sum(stage_avg[k] for k in prep_stages) / 1e3
    prep_gbs = sum(alg_bytes[STAGES[k]] for k in prep_stages) / prep_t / 1e9
    prep_hbm = {"achieved": prep_gbs, "peak": hbm, "unit": "GB/s", "frac": prep_gbs / hbm,
                "stages": [STAGES[k] for k in prep_stages], "ms": prep_t * 1e3}

    # End to end through the public API with pinned host buffers: every step copies its q, k, v
    # host to device, runs the call and copies O back. Steps are pipelined as a serving loop
    # would run them: two device buffer sets, the H2D copies on one stream, the calls on
    # another, the D2H copies on a third, so step i + 1's inputs cross PCIe while step i
    # computes and step i's output returns during step i + 1. Every step's copies stay inside
    # the timed region.
    e2e = None
    if rank == 0 or world > 1:
        hq, hk, hv = (t.pin_memory() for t in (w.q, w.k, w.v))
        ho = torch.empty(w.q.shape, dtype=w.q.dtype).pin_memory()
        sets = [(qs[0], ks[0], vs[0], outs[0])]
        sets.append((torch.empty_like(qs[0]), torch.empty_like(ks[0]), torch.empty_like(vs[0]),
                     torch.empty_like(outs[0])))
        dws = wss[0]
        s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                b = i & 1
                dq, dk, dv, do = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_cmp[b])  # the call two steps back has read this set
                    dq.copy_(hq, non_blocking=True); dk.copy_(hk, non_blocking=True); dv.copy_(hv, non_blocking=True)
                    ev_in[b].record(s_in)
                s_cmp.wait_event(ev_in[b])
                if i >= 2:
                    s_cmp.wait_event(ev_out[b])  # this set's previous output has been copied out
                ba.attention_fwd(dq, dk, dv, bias, out=do, workspace=dws, stream=s_cmp)
                ev_cmp[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[b])
                    ho.copy_(do, non_blocking=True)
                    ev_out[b].record(s_out)

        e2e_steps(2)
        torch.cuda.synchronize()
        ne = max(2, args.e2e_steps)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        s_cmp.wait_event(a0)
        s_out.wait_event(a0)
        e2e_steps(ne)
        s_out.wait_stream(s_cmp)
        s_out.wait_stream(s_in)
        a1.record(s_out)
        torch.cuda.synchronize()
        e_ms = a0.elapsed_time(a1) / ne
        if world > 1:
            e_ms = max_over_ranks(e_ms, dist, dev)
        e2e = {"value": job_throughput(ops, tokens, e_ms, world)[0], "unit": UNIT,
               "h2d_bytes_per_step": 3 * E * esz, "d2h_bytes_per_step": E * esz, "ms_per_step": e_ms,
               "pipelined": "two buffer sets; step i + 1's H2D and step i's D2H overlap step i's call"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        c_ops, c_s, desc = oracle_sample(w, args.cpu_seconds, threads)
        cpu = {"value": c_ops / c_s / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    if ba.kv_block() != workload_config(w)["kv_block"]:
        raise RuntimeError("library key block differs from the quantisation contract's 128")
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {**workload_config(w), "attn_kernel": impl_used, "parallelism": f"replicas x{world}",
                       "l2": f"{R} rotating input sets of {set_bytes / 2**20:.0f} MiB (cycle > 126 MB L2)"},
            "tokens_per_s": tok_s,
            "pct_int8_peak": 100.0 * value / (world * int8_tops),
            "attention_kernel_ms": attn_ms,
            "attention_kernel_tops": ops / (attn_ms / 1e3) / 1e12 if attn_ms > 0 else None,
            "stage_ms": dict(zip(STAGES, stage_avg)),
            "prep_hbm": prep_hbm,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            # prep (1 launch on the one-launch path, else streaming + quantiser) + attention
            "gpu_launches": ((2 if ba.prep_fused(w.B, w.H, w.N, w.d) else 3) * args.steps),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
