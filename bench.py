"""LoRA-MLP fwd+bwd throughput on B200 (tokens/s at the Llama-3-8B MLP shape).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 8b|8b-4bit|1b|tiny]

One step = RMSNorm -> gate/up(+LoRA) -> SwiGLU -> down(+LoRA) forward and the
hand-derived backward (dX and the six adapter gradients) over one batch of
T = 8192 tokens (batch 4 x seq 2048), d = 4096, f = 14336, r = 16, alpha = 16,
on seeded synthetic bf16 inputs.  With N > 1 (one process per GPU, launched by
torchrun, or by this script itself when started without it) every rank runs its own
batch (weak scaling) and the adapter gradients are summed across ranks with one NCCL
all-reduce per step, as data-parallel LoRA training does.  Rank 0 prints one JSON line.

The default line also carries sub-records measured in the same run on the same GPU:
the Llama-3.2-1B MLP shape, the 8B shape with 4-bit frozen weights, and the 8B model's
attention Q/K/V projections, o_proj, RoPE and LM-head cross-entropy, each with its
dominant kernel's fraction of its roofline.

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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LoRA-MLP fwd+bwd tokens/s at Llama-3-8B shape; % of bf16 tensor-core peak"
UNIT = "tokens/s"
CODEBOOK_FILE = os.path.join(ROOT, "tests", "golden", "codebook16.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
KERNEL_SOURCES = ("gemm_sm100.cuh", "ptx.cuh", "host.cuh", "lora_mlp.cu")
GEMM_PHASES = ("gemm_gate_up_swiglu", "gemm_down", "gemm_dact_swiglu_bwd", "gemm_dH")


def peaks():
    """Roofline denominators: MEASURED_PEAKS.json when present (measured on this
    pool's B200s), else the recorded fallback of this pool."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return {"hbm": float(j.get("hbm_gbs", 6650.0)), "burst": float(j.get("bf16_tflops", 1590.0)),
                "sustained": float(j.get("bf16_tflops_sustained", 1400.0)), "source": "measured", "raw": j}
    return {"hbm": 6650.0, "burst": 1590.0, "sustained": 1400.0, "source": "fallback", "raw": {}}


def load_codebook():
    """The 16-entry 4-bit codebook (an input of the 4-bit kernels, stored by the oracle's
    writer script)."""
    with open(CODEBOOK_FILE) as fh:
        return [float.fromhex(h) for h in json.load(fh)["codebook_f32_hex"]]


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


def dtype_for(config):
    return "bf16 activations, 4-bit codebook weights (block 64, fp32 absmax)" if config == "8b-4bit" else "bf16"


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
REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """Samples the SM clock, power and clock-event reasons of one GPU every ~2 ms with
    read-only NVML queries in a background thread; `window(label)` marks a timed region
    and `stats(label)` summarises the samples taken inside it."""

    def __init__(self, cuda_index, period_s=0.002):
        self.samples, self.windows, self.period = [], {}, period_s
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                pr = torch.cuda.get_device_properties(cuda_index)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return
        self.stop_ev = threading.Event()
        self.th = threading.Thread(target=self._run, daemon=True)
        self.th.start()

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1e3, self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    class _Win:
        def __init__(self, owner, label):
            self.owner, self.label = owner, label

        def __enter__(self):
            self.t0 = time.perf_counter()

        def __exit__(self, *exc):
            self.owner.windows.setdefault(self.label, []).append((self.t0, time.perf_counter()))

    def window(self, label):
        return ClockSampler._Win(self, label)

    def stats(self, *labels):
        if not self.ok:
            return None
        spans = [w for lb in labels for w in self.windows.get(lb, [])]
        rows = [s for s in list(self.samples) if any(a <= s[0] <= b for a, b in spans)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
        mask = 0
        for s in rows:
            mask |= s[3]
        return {"sm_mhz": statistics.median(s[1] for s in rows), "sm_min_mhz": min(s[1] for s in rows),
                "sm_max_mhz": self.max_mhz, "power_w_median": statistics.median(s[2] for s in rows),
                "reasons": sorted(n for b, n in REASON_BITS.items() if mask & b), "samples": len(rows),
                "source": "nvml, ~2 ms period, during the timed region"}

    def stop(self):
        if self.ok:
            self.stop_ev.set()
            self.th.join(timeout=2)


# ------------------------------------------------------------------ timing
def timed(step, steps, stream, clk=None, label=None, phases=False):
    """Events around `steps` calls of step() on `stream` (after a synchronize); returns
    total ms and, with `phases`, the library's per-phase times of those calls (their
    events are off otherwise, so a plain timed loop carries none)."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import ops
    ops.timing_enable(phases)
    ops.timing_collect()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = clk.window(label) if clk else None
    if ctx:
        ctx.__enter__()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if ctx:
        ctx.__exit__(None, None, None)
    ph = ops.timing_collect() if phases else {}
    ops.timing_enable(False)
    return e0.elapsed_time(e1), ph


def timed_with_phases(step, steps, stream, clk=None, label=None):
    """The timed loop (no phase events; clocks sampled), then the same number of steps
    again with the phase events on for the per-kernel breakdown."""
    ms, _ = timed(step, steps, stream, clk, label)
    _, ph = timed(step, steps, stream, phases=True)
    return ms, ph


def dominant(phases, name, flops_per_step, steps, peak):
    """Achieved rate of the launches of phase `name`: their algorithmic FLOPs per step
    (all launches of the phase in one step) over their summed time per step."""
    ms, n = phases.get(name, (0.0, 0))
    if not n:
        return None
    ach = flops_per_step / (ms / steps / 1e3) / 1e12
    return {"kernel": name, "achieved_tflops": ach, "frac_of_burst": ach / peak, "launches_per_step": n / steps,
            "us_per_step": 1e3 * ms / steps}


def sub_records(args, pb8, bits8, clk, pk):
    """The other workloads, measured on the same GPU in the same run (fresh buffers each;
    the 4-bit record re-quantises the 8B problem's frozen weights in place)."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import CeProblem, OProblem, Problem, QkvProblem, RopeProblem
    out = {}
    steps = max(5, min(args.steps, 20))
    stream = torch.cuda.current_stream()

    def rec(label, workload, shape_T, flops, ms, ph, dom_name, dom_flops, dtype="bf16"):
        out[label] = {"workload": workload, "dtype": dtype, "steps": steps, "warmup": 3, "ms_per_step": ms / steps,
                      "tokens_per_s": shape_T * steps / (ms / 1e3), "tflops": flops * steps / (ms / 1e3) / 1e12,
                      "dominant": dominant(ph, dom_name, dom_flops, steps, pk["burst"]),
                      "gpu_launches": sum(n for _, n in ph.values()), "clocks": clk.stats(label) if clk else None}

    # Llama-3.2-1B MLP shape
    s1 = configs.LLAMA32_1B
    pb = Problem(s1, synth.make_inputs_bits(s1))
    for _ in range(3):
        pb.step()
    ms, ph = timed_with_phases(pb.step, steps, stream, clk, "config_1b")
    rec("config_1b", f"LoRA-MLP fwd+bwd, Llama-3.2-1B MLP shape: T={s1.T} d={s1.d} f={s1.f} r={s1.r} alpha=16",
        s1.T, configs.algorithmic_flops(s1), ms, ph, "gemm_gate_up_swiglu",
        4.0 * s1.T * s1.d * s1.f + 4.0 * s1.T * s1.r * s1.f)
    del pb
    # 8B shape, 4-bit frozen weights (quantised on the GPU: one-off set-up, not timed)
    s8 = pb8.shape
    pb8.use_4bit(load_codebook(), drop_bf16=False)
    for _ in range(3):
        pb8.step()
    ms, ph = timed_with_phases(pb8.step, steps, stream, clk, "config_4bit")
    rec("config_4bit", f"LoRA-MLP fwd+bwd, Llama-3-8B MLP shape with 4-bit frozen W (block 64): T={s8.T} d={s8.d} "
        f"f={s8.f} r={s8.r} alpha=16", s8.T, configs.algorithmic_flops(s8), ms, ph, "gemm_gate_up_swiglu",
        4.0 * s8.T * s8.d * s8.f + 4.0 * s8.T * s8.r * s8.f, dtype=dtype_for("8b-4bit"))
    # the same with double-quantised block constants (8-bit codes + an fp32 scale per 256)
    pb8.use_4bit(load_codebook(), double_quant=True)
    for _ in range(3):
        pb8.step()
    ms, ph = timed_with_phases(pb8.step, steps, stream, clk, "config_4bit_dq")
    rec("config_4bit_dq", f"LoRA-MLP fwd+bwd, Llama-3-8B MLP shape with 4-bit frozen W, double-quantised block "
        f"constants: T={s8.T} d={s8.d} f={s8.f} r={s8.r} alpha=16", s8.T, configs.algorithmic_flops(s8), ms, ph,
        "gemm_gate_up_swiglu", 4.0 * s8.T * s8.d * s8.f + 4.0 * s8.T * s8.r * s8.f,
        dtype="bf16 activations, 4-bit codebook weights, 8-bit block constants")
    # attention Q/K/V projections of the 8B model
    sq = configs.QKV_8B
    qp = QkvProblem(sq)
    for _ in range(3):
        qp.step()
    ms, ph = timed_with_phases(qp.step, steps, stream, clk, "qkv")
    rec("qkv", f"LoRA Q/K/V projections fwd+bwd, Llama-3-8B attention shape: T={sq.T} d={sq.d} nq={sq.nq} "
        f"nkv={sq.nkv} r={sq.r} alpha=16", sq.T, configs.qkv_algorithmic_flops(sq), ms, ph, "qkv_gemm",
        2.0 * sq.T * sq.d * (sq.nq + 2 * sq.nkv))
    del qp
    # attention output projection o_proj of the 8B model
    so = configs.O_8B
    op = OProblem(so)
    for _ in range(3):
        op.step()
    ms, ph = timed_with_phases(op.step, steps, stream, clk, "o_proj")
    rec("o_proj", f"LoRA o_proj fwd+bwd, Llama-3-8B shape: T={so.T} n_in={so.n_in} n_out={so.n_out} r={so.r} "
        "alpha=16", so.T, configs.o_algorithmic_flops(so), ms, ph, "o_gemm", 2.0 * so.T * so.n_in * so.n_out)
    del op
    # RoPE on the 8B model's query / key heads (forward + backward, in place)
    sr = configs.ROPE_8B
    rp = RopeProblem(sr)
    for _ in range(3):
        rp.step()
    ms, ph = timed_with_phases(rp.step, steps, stream, clk, "rope")
    rb = configs.rope_bytes(sr)
    rms, rn = ph.get("rope", (0.0, 0))
    gbs = rb / (rms / rn / 1e3) / 1e9 if rn else None
    out["rope"] = {"workload": f"RoPE fwd+bwd on Q/K in place, Llama-3-8B heads: T={sr.T} hq={sr.hq} hk={sr.hk} "
                               f"hd={sr.hd} seq={sr.seq_len} base={sr.base:g}",
                   "dtype": "bf16 (fp32 tables)", "steps": steps, "warmup": 3, "ms_per_step": ms / steps,
                   "tokens_per_s": sr.T * steps / (ms / 1e3),
                   "dominant": {"kernel": "rope", "bytes_per_launch": rb, "GB/s": gbs,
                                "frac_of_hbm": gbs / pk["hbm"] if gbs else None,
                                "us_per_launch": 1e3 * rms / rn if rn else None},
                   "gpu_launches": sum(n for _, n in ph.values()), "clocks": clk.stats("rope") if clk else None}
    del rp
    # fused LM-head cross-entropy of the 8B model (vocabulary 128256)
    sc = configs.CE_8B
    cp = CeProblem(sc)
    for _ in range(3):
        cp.step()
    ms, ph = timed_with_phases(cp.step, steps, stream, clk, "ce")
    rec("ce", f"fused LM-head cross-entropy fwd+bwd, Llama-3-8B head: T={sc.T} d={sc.d} V={sc.V} "
        f"(vocabulary chunk 32768 in the backward)", sc.T, configs.ce_algorithmic_flops(sc), ms, ph,
        "ce_gemm_lse", 2.0 * sc.T * sc.d * sc.V)
    del cp
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ our arm
def ours_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
    from lora_fine_tuning_rmsnorm_b200 import dist as ldist
    from lora_fine_tuning_rmsnorm_b200.runner import GRADS, HostPipeline, Problem, bf16_tensor

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
    barrier()
    ms, _ = timed(step, args.steps, stream, clk, "main")
    barrier()
    ms = ldist.max_over_ranks(ms, dev)
    # per-kernel breakdown: the same number of steps again with the library's phase events
    # on (outside the timed region; every rank takes the same steps)
    _, phases = timed(step, args.steps, stream, phases=True)
    value = world * shape.T * args.steps / (ms / 1e3)

    # ---- end-to-end through the C ABI with host buffers (pinned): every step copies its
    # inputs in and its results (Y, dX, gradients) out inside the timed region; the copies
    # are double-buffered, one stream per direction, and overlap the neighbouring steps' compute
    hX = bf16_tensor(bits["X"], "cpu", pin=True)
    hdY = bf16_tensor(bits["dY"], "cpu", pin=True)
    pipe = HostPipeline(pb, hX, hdY, reduce=ldist.allreduce_grads if world > 1 else None)
    pipe.start()
    for i in range(2):
        pipe.step(i, 2)
    torch.cuda.synchronize(dev)
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    win = clk.window("e2e") if clk else None
    if win:
        win.__enter__()
    f0.record(pipe.xs)
    pipe.start()
    for i in range(args.steps):
        pipe.step(i, args.steps)
    pipe.finish()
    f1.record(pipe.xs)
    torch.cuda.synchronize(dev)
    if win:
        win.__exit__(None, None, None)
    barrier()
    ms_e2e = ldist.max_over_ranks(f0.elapsed_time(f1), dev)
    e2e_value = world * shape.T * args.steps / (ms_e2e / 1e3)
    h2d, d2h = pipe.h2d_bytes, pipe.d2h_bytes
    del pipe

    pk = peaks()
    subs = {}
    if world == 1 and args.config == "8b" and not args.no_sub and args.T is None:
        subs = sub_records(args, pb, bits, clk, pk)
    if clk:
        clk.stop()
    if rank != 0:
        return
    T, d, f, r = shape.T, shape.d, shape.f, shape.r
    # dominant kernel: the dense GEMM with the most time per step (gate/up and dH are within a
    # few per cent of each other at the 8B shape), with its algorithmic FLOPs per launch
    gemm_flops_per_launch = {"gemm_gate_up_swiglu": 4.0 * T * d * f + 4.0 * T * r * f,
                             "gemm_down": 2.0 * T * d * f + 2.0 * T * r * d,
                             "gemm_dact_swiglu_bwd": 2.0 * T * d * f + 2.0 * T * r * f,
                             "gemm_dH": 4.0 * T * d * f + 4.0 * T * r * d}
    dom = max(GEMM_PHASES, key=lambda k: phases.get(k, (0.0, 0))[0])
    dom_ms, dom_n = phases.get(dom, (0.0, 0))
    dom_flops = gemm_flops_per_launch[dom]
    dom_tflops = dom_flops / (dom_ms / dom_n / 1e3) / 1e12 if dom_n else None
    flops = configs.algorithmic_flops(shape)
    step_ms = ms / args.steps
    gemm_ms = sum(phases.get(k, (0.0, 0))[0] for k in GEMM_PHASES) / args.steps
    gemm_flops = 12.0 * T * d * f + 4.0 * T * r * f + 2.0 * T * r * d + 2.0 * T * r * f + 4.0 * T * r * d
    rms_fwd_ms = phases.get("rmsnorm_fwd", (0.0, 1))[0] / args.steps
    rms_bwd_ms = phases.get("rmsnorm_bwd", (0.0, 1))[0] / args.steps
    rms_fwd_bytes = T * (4 * d + 4)
    rms_bwd_bytes = T * (8 * d + 4)
    launches = sum(n for _, n in phases.values())
    clocks = clk.stats("main", "e2e") if clk else None
    roof = {"bound": "tensor", "kernel": dom, "achieved": dom_tflops, "peak": pk["burst"], "unit": "TFLOP/s",
            "frac": (dom_tflops / pk["burst"]) if dom_tflops else None,
            "traffic": measured_traffic(dom, args.config),
            "peak_source": f"bf16_tflops burst ({pk['source']}): the timed region lasts well under a second",
            "flops_per_launch": dom_flops, "frac_of_sustained": (dom_tflops / pk["sustained"]) if dom_tflops else None}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_for(args.config),
        "data": "synthetic (seeded; bf16 weights/activations, fp32 accumulate)",
        "config": config_for(args, shape, world),
        "tflops": flops / (step_ms / 1e3) / 1e12,
        "pct_bf16_peak": flops / (step_ms / 1e3) / 1e12 / pk["burst"],
        "roofline": roof,
        "phase_rooflines": {
            "gemm_phases_frac_of_bf16_burst": gemm_flops / (gemm_ms / 1e3) / 1e12 / pk["burst"] if gemm_ms else None,
            "rmsnorm_fwd_frac_of_hbm": rms_fwd_bytes / (rms_fwd_ms / 1e3) / 1e9 / pk["hbm"] if rms_fwd_ms else None,
            "rmsnorm_bwd_frac_of_hbm": rms_bwd_bytes / (rms_bwd_ms / 1e3) / 1e9 / pk["hbm"] if rms_bwd_ms else None,
        },
        "phases_ms_per_step": {k: v[0] / args.steps for k, v in sorted(phases.items())},
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
        "peaks": {k: pk[k] for k in ("hbm", "burst", "sustained", "source")},
    }
    if clocks and clocks.get("sm_mhz") and pk["raw"]:
        mhz = [v for k, v in pk["raw"].items() if "mhz" in k.lower() and "bf16" in k.lower()
               and isinstance(v, (int, float))]
        if mhz and dom_tflops:
            # the same kernel time rescaled to the clock the burst peak was measured at
            roof["frac_clock_normalised"] = dom_tflops * (mhz[0] / clocks["sm_mhz"]) / pk["burst"]
    line.update(subs)
    if world == 1 and not args.no_cpu_baseline:
        ot = OracleTimer(shape, bits, max_rows=shape.T)
        n = ot.size_for(12.0)
        t = ot.run(n)
        line["cpu_baseline"] = {"value": n / t, "unit": UNIT, "cores": ot.cores, "kind": "oracle",
                                "sample": f"{n} of {T} rows, fp64 NumPy oracle fwd+bwd over all weights ({t:.1f} s)"}
    print(json.dumps(line), flush=True)


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
    """DRAM bytes per launch of `kernel` from the committed ncu record (a JSON list), if
    it was taken on the current kernel sources; None otherwise."""
    try:
        with open(TRAFFIC_FILE) as fh:
            recs = json.load(fh)["records"]
    except (OSError, ValueError, KeyError):
        return None
    digest = sources_digest()
    for rec in recs:
        if rec.get("kernel") == kernel and rec.get("config") == config and rec.get("sources") == digest:
            return float(rec["bytes_per_launch"])
    return None


def extras(args):
    """The variants around the path at the 8B shape, one JSON line: a step with the
    residual connection and the norm-weight gradient against the plain step, the dw
    kernel and the weight merge of a [f x d] matrix against the HBM roofline."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import Problem
    torch.cuda.set_device(0)
    hbm = peaks()["hbm"]
    shape = shape_for("8b", args.T)
    T, d, f, r = shape.T, shape.d, shape.f, shape.r
    bits = synth.make_inputs_bits(shape)
    out = {"extras": True, "config": config_for(args, shape, 1)}
    stream = torch.cuda.current_stream()

    def timed_steps(pb):
        for _ in range(args.warmup):
            pb.step()
        ms, ph = timed_with_phases(pb.step, args.steps, stream)
        return ms / args.steps, ph

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


def sweep(args):
    """Rank / length sweep at d = 4096, f = 14336 (alpha = 16): one JSON line per
    point with tokens/s and the dense-GEMM vs memory-bound phase split."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import configs, synth
    from lora_fine_tuning_rmsnorm_b200.runner import Problem
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    for s in configs.SWEEP:
        pb = Problem(s, synth.make_inputs_bits(s))
        for _ in range(args.warmup):
            pb.step()
        ms, ph = timed_with_phases(pb.step, args.steps, stream)
        ms /= args.steps
        gemm = sum(ph.get(k, (0.0, 0))[0] for k in GEMM_PHASES) / args.steps
        other = sum(v[0] for k, v in ph.items() if k not in GEMM_PHASES) / args.steps
        print(json.dumps({"sweep": True, "T": s.T, "r": s.r, "tokens_per_s": s.T / (ms / 1e3), "ms_per_step": ms,
                          "tflops": configs.algorithmic_flops(s) / (ms / 1e3) / 1e12,
                          "gemm_ms": gemm, "memory_bound_ms": other}), flush=True)
        del pb
        torch.cuda.empty_cache()


def stub_arm(args, rank, world):
    """CPU check of the multi-rank plumbing (gloo): the same launcher, process group,
    max-over-ranks timing and flat-buffer all-reduce as the GPU arm, around a stub step
    whose 'time' and gradients depend on the rank."""
    import datetime

    import torch
    import torch.distributed as dist

    from lora_fine_tuning_rmsnorm_b200 import dist as ldist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        flat, views = ldist.flat_grads(16, 24, 8)
        ok = True
        for _ in range(args.warmup + args.steps):
            flat.fill_(float(rank + 1))
            ldist.allreduce_grads(flat)
            ok = ok and bool(torch.all(flat == world * (world + 1) / 2))
        ms = ldist.max_over_ranks(10.0 * (rank + 1), torch.device("cpu"))
        if rank == 0:
            print(json.dumps({"stub": True, "n_gpus": world, "ms_max_over_ranks": ms, "allreduce_ok": ok,
                              "value": world * 1000 * args.steps / (ms / 1e3), "unit": UNIT}), flush=True)
    finally:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="8b", choices=["8b", "8b-4bit", "1b", "tiny"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample the clocks (profiling runs)")
    ap.add_argument("--no-sub", action="store_true", help="skip the 1B / 4-bit / Q/K/V sub-records")
    ap.add_argument("--T", type=int, default=None, help="override the token count (profiling on small cases)")
    ap.add_argument("--sweep", action="store_true", help="rank/length sweep, one JSON line per point")
    ap.add_argument("--extras", action="store_true",
                    help="residual / norm-weight-gradient step and weight merge, one JSON line")
    ap.add_argument("--stub-cpu", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start this script again under torchrun with the same flags
        from lora_fine_tuning_rmsnorm_b200 import dist as ldist
        cmd = ldist.torchrun_argv(args.gpus, os.path.abspath(__file__), sys.argv[1:])
        sys.exit(subprocess.run(cmd, timeout=1800).returncode)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 and world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.stub_cpu:
        stub_arm(args, rank, world)
        return
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if args.sweep:
        sweep(args)
        return
    if args.extras:
        extras(args)
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
