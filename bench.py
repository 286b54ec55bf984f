"""LoRA-MLP fwd+bwd throughput on B200 (tokens/s at the Llama-3-8B MLP shape).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 8b|1b|tiny]

One step = RMSNorm -> gate/up(+LoRA) -> SwiGLU -> down(+LoRA) forward and the
hand-derived backward (dX and the six adapter gradients) over one batch of
T = 8192 tokens (batch 4 x seq 2048), d = 4096, f = 14336, r = 16, alpha = 16,
on seeded synthetic bf16 inputs.  With N > 1 (one process per GPU under torchrun)
every rank runs its own batch (weak scaling) and the adapter gradients are summed
across ranks with one NCCL all-reduce per step, as data-parallel LoRA training
does.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on this host's cores instead (a bounded
sample of rows per step), on the same metric and unit.
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

METRIC = "LoRA-MLP fwd+bwd tokens/s at Llama-3-8B shape; % of bf16 tensor-core peak"
UNIT = "tokens/s"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return j.get("hbm_gbs", 6650.0), j.get("bf16_tflops", 1590.0), j.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def shape_for(name, T=None):
    import dataclasses
    from lora_fine_tuning_rmsnorm_b200 import configs
    s = {"8b": configs.LLAMA3_8B, "8b-4bit": configs.LLAMA3_8B, "1b": configs.LLAMA32_1B,
         "tiny": configs.TINY}[name]
    return dataclasses.replace(s, T=T) if T else s


# ------------------------------------------------------------------ CPU oracle
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return len(os.sched_getaffinity(0))


class OracleTimer:
    """Times the fp64 oracle (as it stands) fwd+bwd on a bounded sample of rows."""

    def __init__(self, shape, bits=None, max_rows=2048):
        from lora_fine_tuning_rmsnorm_b200 import synth
        self.shape = shape
        if bits is None:
            bits = synth.make_inputs_bits(synth.Shape(T=min(shape.T, max_rows), d=shape.d, f=shape.f, r=shape.r,
                                                      alpha=shape.alpha, eps=shape.eps))
        self.inp = synth.bits_to_f64({k: (v[:max_rows] if k in ("X", "dY") else v) for k, v in bits.items()})
        self.cores = _blas_threads()

    def run(self, n):
        from oracle import lora_mlp_ref as ref
        sub = dict(self.inp)
        sub["X"], sub["dY"] = self.inp["X"][:n], self.inp["dY"][:n]
        t0 = time.perf_counter()
        ref.fwd_bwd(sub, self.shape.scale, self.shape.eps, chunk=1024, keep=("Y", "dX"))
        return time.perf_counter() - t0

    def size_for(self, target_s):
        n = 64
        t = self.run(n)
        n = int(n * target_s / max(t, 1e-3))
        return max(16, min(n, len(self.inp["X"])))


def config_for(args, shape, world):
    """The workload description both arms print (same sizes, same wording)."""
    T, d, f, r = shape.T, shape.d, shape.f, shape.r
    if args.config in ("8b", "8b-4bit"):
        wl = (f"LoRA-MLP fwd+bwd, Llama-3-8B MLP shape: T={T} (batch 4 x seq 2048) d={d} f={f} "
              f"r={r} alpha={shape.alpha:g}" + (", 4-bit frozen W (blocksize 64)" if args.config == "8b-4bit" else ""))
    else:
        wl = f"LoRA-MLP fwd+bwd {args.config}: T={T} d={d} f={f} r={r}"
    return {"workload": wl, "global_batch": T * world, "seq_len": 2048, "parallelism": f"dp{world}",
            "l2": "inputs larger than L2 (weights 336 MB + activations), no flush"}


def reference_arm(args, rank, world):
    if rank != 0:
        return
    shape = shape_for(args.config)
    ot = OracleTimer(shape)
    n = ot.size_for(max(1.0, 90.0 / (args.steps + args.warmup)))
    times = []
    for i in range(args.warmup + args.steps):
        t = ot.run(n)
        if i >= args.warmup:
            times.append(t)
    t_med = statistics.median(times)
    value = n / t_med
    sample = f"{n} of {shape.T} rows per step (fp64 NumPy oracle fwd+bwd over all weights)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_med,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, bf16-rounded)",
        "config": config_for(args, shape, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": ot.cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index):
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"lora_mlp_clocks_{os.getpid()}.csv")
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for ln in open(self.path):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ our arm
def ours_arm(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
    from lora_fine_tuning_rmsnorm_b200 import dist as ldist
    from lora_fine_tuning_rmsnorm_b200.runner import GRADS, HostPipeline, Problem, bf16_tensor, load_codebook

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    shape = shape_for(args.config, args.T)
    bits = synth.make_inputs_bits(shape)
    pb = Problem(shape, bits, device=dev)
    if args.config == "8b-4bit":
        pb.use_4bit(load_codebook())  # one-off quantisation of the frozen weights (set-up)
    # one flat fp32 buffer for the six adapter gradients -> one all-reduce per step
    flat, views = ldist.flat_grads(shape.d, shape.f, shape.r, device=dev)
    pb.g = views
    pb.grads = ops.make_grads(*(pb.g[k] for k in GRADS))
    stream = torch.cuda.current_stream(dev)

    def step():
        pb.forward(stream=stream)
        pb.backward(stream=stream)
        ldist.allreduce_grads(flat)

    def barrier():
        if world > 1:
            dist.barrier()

    clk = ClockSampler(local_rank) if (rank == 0 and not args.no_clocks) else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # ---- device-resident timed region
    ops.timing_enable(True)
    ops.timing_collect()
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1)
    phases = ops.timing_collect()
    ops.timing_enable(False)

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    ms = max_over_ranks(ms)
    tokens = world * shape.T * args.steps
    value = tokens / (ms / 1e3)

    # ---- end-to-end through the C ABI with host buffers (pinned): every step copies its
    # inputs in and its results (Y, dX, gradients) out inside the timed region; the copies
    # are double-buffered on a second stream and overlap the neighbouring steps' compute
    hX = bf16_tensor(bits["X"], "cpu", pin=True)
    hdY = bf16_tensor(bits["dY"], "cpu", pin=True)
    pipe = HostPipeline(pb, hX, hdY, reduce=ldist.allreduce_grads if world > 1 else None)
    pipe.start()
    for i in range(2):
        pipe.step(i, 2)
    torch.cuda.synchronize(dev)
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(pipe.xs)
    pipe.start()
    for i in range(args.steps):
        pipe.step(i, args.steps)
    f1.record(pipe.xs)
    torch.cuda.synchronize(dev)
    barrier()
    ms_e2e = max_over_ranks(f0.elapsed_time(f1))
    e2e_value = world * shape.T * args.steps / (ms_e2e / 1e3)
    clocks = clk.stop() if clk else None
    h2d = pipe.h2d_bytes
    d2h = pipe.d2h_bytes

    if rank != 0:
        return
    hbm, bf16_burst, bf16_sust, src = peaks()
    T, d, f, r = shape.T, shape.d, shape.f, shape.r
    # dominant kernel: the gate/up GEMM with the LoRA B-term and the SwiGLU epilogue
    dom = "gemm_gate_up_swiglu"
    dom_ms, dom_n = phases.get(dom, (0.0, 0))
    dom_flops = 4.0 * T * d * f + 4.0 * T * r * f
    dom_tflops = dom_flops / (dom_ms / dom_n / 1e3) / 1e12 if dom_n else None
    flops = configs.algorithmic_flops(shape)
    step_ms = ms / args.steps
    gemm_names = ("gemm_gate_up_swiglu", "gemm_down", "gemm_dact_swiglu_bwd", "gemm_dH")
    gemm_ms = sum(phases.get(k, (0.0, 0))[0] for k in gemm_names) / args.steps
    gemm_flops = 12.0 * T * d * f + 4.0 * T * r * f + 2.0 * T * r * d + 2.0 * T * r * f + 4.0 * T * r * d
    rms_fwd_ms = phases.get("rmsnorm_fwd", (0.0, 1))[0] / args.steps
    rms_bwd_ms = phases.get("rmsnorm_bwd", (0.0, 1))[0] / args.steps
    rms_fwd_bytes = T * (4 * d + 4)
    rms_bwd_bytes = T * (8 * d + 4)
    launches = sum(n for _, n in phases.values())
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; bf16 weights/activations, fp32 accumulate)",
        "config": config_for(args, shape, world),
        "tflops": flops / (step_ms / 1e3) / 1e12,
        "pct_bf16_peak": flops / (step_ms / 1e3) / 1e12 / bf16_sust,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": dom_tflops, "peak": bf16_sust,
                     "unit": "TFLOP/s", "frac": (dom_tflops / bf16_sust) if dom_tflops else None,
                     "traffic": measured_traffic(dom, args.config),
                     "peak_source": f"bf16_tflops_sustained ({src})",
                     "flops_per_launch": dom_flops},
        "phase_rooflines": {
            "gemm_phases_frac_of_bf16_sustained": gemm_flops / (gemm_ms / 1e3) / 1e12 / bf16_sust if gemm_ms else None,
            "rmsnorm_fwd_frac_of_hbm": rms_fwd_bytes / (rms_fwd_ms / 1e3) / 1e9 / hbm if rms_fwd_ms else None,
            "rmsnorm_bwd_frac_of_hbm": rms_bwd_bytes / (rms_bwd_ms / 1e3) / 1e9 / hbm if rms_bwd_ms else None,
        },
        "phases_ms_per_step": {k: v[0] / args.steps for k, v in sorted(phases.items())},
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        ot = OracleTimer(shape, bits, max_rows=shape.T)
        n = ot.size_for(12.0)
        t = ot.run(n)
        line["cpu_baseline"] = {"value": n / t, "unit": UNIT, "cores": ot.cores, "kind": "oracle",
                                "sample": f"{n} of {T} rows, fp64 NumPy oracle fwd+bwd over all weights ({t:.1f} s)"}
    print(json.dumps(line), flush=True)


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_lora_mlp_8b.md")
KERNEL_SOURCES = ("gemm_sm100.cuh", "ptx.cuh", "lora_mlp.cu")


def sources_digest() -> str:
    """sha256 over the code (comments and blank space removed) of the sources the GEMM
    kernels and their launches are built from."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "lora_fine_tuning_rmsnorm_b200", "csrc", name)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, config: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken
    on the current kernel sources (a `traffic-record:` line); None otherwise."""
    try:
        lines = open(TRAFFIC_FILE).read().splitlines()
    except OSError:
        return None
    digest = sources_digest()
    for ln in lines:
        if "traffic-record:" not in ln:
            continue
        kv = dict(x.split("=", 1) for x in ln.split("traffic-record:", 1)[1].split() if "=" in x)
        if kv.get("kernel") == kernel and kv.get("config") == config and kv.get("sources") == digest:
            return float(kv["bytes_per_launch"])
    return None


def extras(args):
    """The variants around the path at the 8B shape, one JSON line: a step with the
    residual connection and the norm-weight gradient against the plain step, the dw
    kernel and the weight merge of a [f x d] matrix against the HBM roofline."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import Problem
    torch.cuda.set_device(0)
    hbm = peaks()[0]
    shape = shape_for("8b", args.T)
    T, d, f, r = shape.T, shape.d, shape.f, shape.r
    bits = synth.make_inputs_bits(shape)
    out = {"extras": True, "config": config_for(args, shape, 1)}

    def timed_steps(pb):
        for _ in range(args.warmup):
            pb.step()
        torch.cuda.synchronize()
        ops.timing_enable(True)
        ops.timing_collect()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            pb.step()
        e1.record()
        torch.cuda.synchronize()
        ph = ops.timing_collect()
        ops.timing_enable(False)
        return e0.elapsed_time(e1) / args.steps, ph

    plain = Problem(shape, bits)
    ms_plain, _ = timed_steps(plain)
    del plain
    var = Problem(shape, bits, residual=True, norm_grad=True)
    ms_var, ph = timed_steps(var)
    dw_ms, dw_n = ph.get("norm_weight_grad", (0.0, 0))
    dw_bytes = T * (4 * d + 2 * d + 4) + 4 * d   # dH fp32 + X bf16 + rstd read, dw written
    dw_gbs = dw_bytes / (dw_ms / dw_n / 1e3) / 1e9 if dw_n else None
    out["residual_and_norm_grad"] = {"ms_per_step": ms_var, "plain_ms_per_step": ms_plain,
                                     "overhead_ms": ms_var - ms_plain}
    out["norm_weight_grad"] = {"us_per_launch": 1e3 * dw_ms / dw_n if dw_n else None, "algorithmic_bytes": dw_bytes,
                               "GB/s": dw_gbs, "frac_of_hbm": dw_gbs / hbm if dw_gbs else None}
    W, A, B = var.t["Wg"], var.t["Ag"], var.t["Bg"]
    Wm = torch.empty_like(W)
    for _ in range(3):
        ops.merge_weights(W, A, B, shape.scale, out=Wm)
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        ops.merge_weights(W, A, B, shape.scale, out=Wm)
    e1.record()
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / reps
    mb = f * d * 4 + (r * d + f * r) * 2          # W read + Wm written (+ A, B)
    out["merge_weights"] = {"rows": f, "cols": d, "r": r, "us_per_launch": us, "algorithmic_bytes": mb,
                            "GB/s": mb / (us / 1e6) / 1e9, "frac_of_hbm": mb / (us / 1e6) / 1e9 / hbm}
    out["hbm_peak_gbs"] = hbm
    print(json.dumps(out), flush=True)


def qkv(args):
    """LoRA Q/K/V projections fwd+bwd at the 8B attention shape: one JSON line with
    tokens/s, algorithmic TFLOP/s and the fraction of the sustained bf16 peak."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import configs
    from lora_fine_tuning_rmsnorm_b200.runner import QkvProblem
    torch.cuda.set_device(0)
    s = configs.QKV_8B if not args.T else configs.QkvShape(T=args.T, d=4096, nq=4096, nkv=1024, r=16)
    pb = QkvProblem(s)
    for _ in range(args.warmup):
        pb.step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        pb.step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    flops = configs.qkv_algorithmic_flops(s)
    sust = peaks()[2]
    print(json.dumps({"qkv": True, "workload": f"LoRA Q/K/V projections fwd+bwd, Llama-3-8B attention shape: T={s.T} "
                                               f"d={s.d} nq={s.nq} nkv={s.nkv} r={s.r} alpha={s.alpha:g}",
                      "tokens_per_s": s.T / (ms / 1e3), "ms_per_step": ms, "tflops": flops / (ms / 1e3) / 1e12,
                      "frac_of_bf16_sustained": flops / (ms / 1e3) / 1e12 / sust, "steps": args.steps,
                      "warmup": args.warmup}), flush=True)


def sweep(args):
    """Rank / length sweep at d = 4096, f = 14336 (alpha = 16): one JSON line per
    point with tokens/s and the dense-GEMM vs memory-bound phase split."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import Problem
    torch.cuda.set_device(0)
    gemm_names = ("gemm_gate_up_swiglu", "gemm_down", "gemm_dact_swiglu_bwd", "gemm_dH")
    for s in configs.SWEEP:
        bits = synth.make_inputs_bits(s)
        pb = Problem(s, bits)
        for _ in range(args.warmup):
            pb.step()
        torch.cuda.synchronize()
        ops.timing_enable(True)
        ops.timing_collect()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            pb.step()
        e1.record()
        torch.cuda.synchronize()
        ph = ops.timing_collect()
        ops.timing_enable(False)
        ms = e0.elapsed_time(e1) / args.steps
        gemm = sum(ph.get(k, (0.0, 0))[0] for k in gemm_names) / args.steps
        other = sum(v[0] for k, v in ph.items() if k not in gemm_names) / args.steps
        print(json.dumps({"sweep": True, "T": s.T, "r": s.r, "tokens_per_s": s.T / (ms / 1e3), "ms_per_step": ms,
                          "tflops": configs.algorithmic_flops(s) / (ms / 1e3) / 1e12,
                          "gemm_ms": gemm, "memory_bound_ms": other}), flush=True)
        del pb
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="8b", choices=["8b", "8b-4bit", "1b", "tiny"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample nvidia-smi (profiling runs)")
    ap.add_argument("--T", type=int, default=None, help="override the token count (profiling on small cases)")
    ap.add_argument("--sweep", action="store_true", help="rank/length sweep, one JSON line per point")
    ap.add_argument("--qkv", action="store_true", help="LoRA Q/K/V projections fwd+bwd, one JSON line")
    ap.add_argument("--extras", action="store_true",
                    help="residual / norm-weight-gradient step and weight merge, one JSON line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if args.sweep:
        sweep(args)
        return
    if args.extras:
        extras(args)
        return
    if args.qkv:
        qkv(args)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        ours_arm(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
