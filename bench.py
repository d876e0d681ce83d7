#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME] [--only-main]

One step = one training pass of the layer over one batch of synthetic tokens: forward (s*x*A^T, then the
fused NF4-dequant + matmul + LoRA GEMM) and backward (s*dY*B, the fused dX GEMM over transposed NF4 tiles,
dA, dB); with N > 1 ranks each rank runs its own batch (data parallel, weak scaling) and the adapter
gradients dA, dB are summed over ranks with NCCL.  The NF4 weight is quantized once before timing (it is
frozen), as in fine-tuning.

Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the launching stream; the L2 is
flushed (256 MiB write) before every step outside the timed interval; barrier + synchronize on both sides
of the timed loop; the result is the max over ranks.  rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference that exists for this layer) on a bounded
sub-batch of the same workload, on the host cores, rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA fused linear fwd+bwd TFLOP/s and % of BF16/HBM roofline at 1 B200"
DEFAULT_WORKLOAD = "attn_2048x4096x4096_r16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS)


# The sources of the layer library (libqlora's qlora.cu translation unit and what it includes): the kernels
# whose counters are recorded under profiles/ are built from these and nothing else.  The format conversions
# (formats.cu, formats.cuh) are a separate translation unit that none of them includes.
LAYER_SOURCES = ("elementwise.cuh", "nf4_table.cuh", "ptx.cuh", "qlora.cu", "umma_gemm.cuh")


def kernel_source_sha() -> str:
    """Hash of the layer kernels' source code (comments and whitespace removed): recorded profiler counters
    stay valid across comment edits and become stale on any code change."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "qlora_fine_tuning_blockwise_b200", "csrc")
    for name in sorted(LAYER_SOURCES):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name)) as f:
                text = f.read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
            text = re.sub(r"//[^\n]*", " ", text)
            h.update(name.encode())
            h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_traffic() -> dict:
    """ncu DRAM bytes per launch recorded under profiles/, valid only for the kernel source they were taken on."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except Exception:
        return {}
    if t.get("source_sha") != kernel_source_sha():
        return {}
    return t.get("kernels", {})


# ------------------------------------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self) -> dict:
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------ distributed


def dist_setup(n_gpus: int):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------ our arm


def flush_l2(buf):
    buf.zero_()


def run_ours(args, rank, world, local, peaks):
    import torch
    import torch.distributed as dist

    from qlora_fine_tuning_blockwise_b200 import build as qbuild
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    from qlora_fine_tuning_blockwise_b200 import ops
    from qlora_fine_tuning_blockwise_b200.parallel import allreduce_adapter_grads

    qbuild.build()
    w = I.WORKLOADS[args.workload]
    d = I.make_linear_inputs(w, seed=0)
    # every rank its own tokens (data parallel); the frozen weight and the adapters are replicas
    if rank:
        d["x"] = I.draw_x(I._streams(1000 + rank), w.M, w.K, w.x_kind)
        d["dy"] = I.draw_dy(w.M, w.N, 2000 + rank)
    dev = torch.device("cuda", local)
    layer = ops.QLoRALinear(torch.from_numpy(d["W"]).to(dev), d["A"].to(dev), d["B"].to(dev), d["s"])
    x = d["x"].to(dev)
    dy = d["dy"].to(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        y, su = layer.forward(x)
        dx, dA, dB = layer.backward(dy, x, su=su)
        if world > 1:
            allreduce_adapter_grads([dA, dB])
        return y, dx, dA, dB

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = ops.launch_count()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush_l2(flush)
            e = ev[i]
            ops.set_profile_events(0, e[2], e[3])
            ops.set_profile_events(1, e[4], e[5])
            e[0].record(stream)
            step()
            e[1].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    ops.set_profile_events(0, None, None)
    ops.set_profile_events(1, None, None)
    launches = ops.launch_count() - launches0
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    fwd_ms = [e[2].elapsed_time(e[3]) for e in ev]
    dx_ms = [e[4].elapsed_time(e[5]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / K
    flops_step = w.flops_fwd + w.flops_bwd
    value = flops_step * world * K / (total_ms * 1e-3) / 1e12

    # dominant kernel: the fused forward or dX GEMM, whichever takes longer on average
    avg_fwd, avg_dx = sum(fwd_ms) / K, sum(dx_ms) / K
    M, N, Kd, r = w.M, w.N, w.K, w.r
    kern = {
        "fused_fwd": {"ms": avg_fwd, "flops": 2 * M * N * Kd + 2 * M * N * r},
        "fused_dx": {"ms": avg_dx, "flops": 2 * M * N * Kd + 2 * M * Kd * r},
    }
    dom = max(kern, key=lambda k: kern[k]["ms"])
    ach = kern[dom]["flops"] / (kern[dom]["ms"] * 1e-3) / 1e12
    traffic = load_traffic().get(dom)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4),
                "peak_source": peaks["source"] + " bf16 burst", "traffic": traffic,
                "kernel_ms": round(kern[dom]["ms"], 4),
                "other_kernel": {k: {"ms": round(v["ms"], 4),
                                     "tflops": round(v["flops"] / (v["ms"] * 1e-3) / 1e12, 1)}
                                 for k, v in kern.items() if k != dom}}
    step_roof_ms = max(flops_step / (peaks["bf16_tflops"] * 1e12), (w.bytes_fwd + w.bytes_bwd) / (peaks["hbm_gbs"] * 1e9)) * 1e3
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "M": M, "N": N, "K": Kd, "r": r, "s": w.s, "tokens_per_rank": M,
                   "global_tokens": M * world, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (256 MiB write, outside the timed interval)"},
        "roofline": roofline,
        "step_roofline_frac": round(step_roof_ms / ms_per_step, 4),
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    return out, (layer, x, dy, d, w, dev)


E2E_RESULTS = {
    # the step's result read back to the host: the adapter gradients, which are what a training step of this
    # layer produces (y and dX are activations that the neighbouring layers consume on the device)
    "grads": ("dA", "dB"),
    # every output of the step
    "all": ("y", "dx", "dA", "dB"),
}


def run_e2e(ctx, args, world, read_back: str = "grads"):
    """Same metric through the public API with host buffers: every step copies its x and dY in from pinned host
    memory and its result out to pinned host memory (``E2E_RESULTS[read_back]``).  Steps are pipelined over three
    streams -- the host-to-device copies of step i + 1 and the device-to-host copies of step i - 1 run while
    step i computes -- with double-buffered device inputs and outputs, ordered by events.  Every step computes
    the whole forward and backward whatever is read back.  The L2 flush runs on the compute stream at the start
    of every step, inside the timed interval.  Time = device time from the first copy in to the last copy out,
    max over ranks."""
    import torch
    import torch.distributed as dist

    from qlora_fine_tuning_blockwise_b200 import ops
    from qlora_fine_tuning_blockwise_b200.parallel import allreduce_adapter_grads

    layer, _x_dev, _dy_dev, d, w, dev = ctx
    x_h = d["x"].pin_memory()
    dy_h = d["dy"].pin_memory()
    M, N, K, r = w.M, w.N, w.K, w.r
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    bufs = layer._buffers(M, dev)  # workspaces: used by the compute stream only, in order
    slots = []
    for _ in range(2):
        slots.append(dict(
            x=torch.empty(M, K, dtype=torch.bfloat16, device=dev),
            dy=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
            y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
            su=torch.empty(M, r, dtype=torch.bfloat16, device=dev) if r else None,
            dx=torch.empty(M, K, dtype=torch.bfloat16, device=dev),
            dA=torch.empty(r, K, dtype=torch.float32, device=dev) if r else None,
            dB=torch.empty(N, r, dtype=torch.float32, device=dev) if r else None,
            h={name: torch.empty(shape, dtype=dt, pin_memory=True)
               for name, shape, dt in (("y", (M, N), torch.bfloat16), ("dx", (M, K), torch.bfloat16),
                                       ("dA", (max(r, 1), K), torch.float32), ("dB", (N, max(r, 1)), torch.float32))},
            in_ready=torch.cuda.Event(), computed=torch.cuda.Event(), out_done=torch.cuda.Event()))
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def issue(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(sl["computed"])  # step i - 2 has finished reading this slot's inputs
            sl["x"].copy_(x_h, non_blocking=True)
            sl["dy"].copy_(dy_h, non_blocking=True)
            sl["in_ready"].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(sl["in_ready"])
            if i >= 2:
                s_comp.wait_event(sl["out_done"])  # step i - 2's outputs have left this slot
            flush_l2(flush)
            ops.qlora_linear_fwd(sl["x"], layer.codes, layer.absmax, layer.A, layer.B, layer.s, N, K,
                                 workspace=bufs["ws_f"], y=sl["y"], su=sl["su"])
            ops.qlora_linear_bwd(sl["dy"], sl["x"], layer.codes, layer.absmax, layer.A, layer.B, layer.s, N, K,
                                 su=sl["su"], workspace=bufs["ws_b"], dx=sl["dx"], dA=sl["dA"], dB=sl["dB"])
            if world > 1:
                allreduce_adapter_grads([sl["dA"], sl["dB"]])
            sl["computed"].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sl["computed"])
            names = [nm for nm in E2E_RESULTS[read_back] if sl[nm] is not None] or ["dx"]  # r = 0: no gradients
            outs = [sl[nm] for nm in names]
            for nm, t in zip(names, outs):
                sl["h"][nm].view(-1)[: t.numel()].copy_(t.view(-1), non_blocking=True)
            sl["out_done"].record(s_out)
        return outs

    for i in range(max(args.warmup, 3)):
        issue(i)
    torch.cuda.synchronize(dev)
    K_steps = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(s_in)
    outs = None
    for i in range(K_steps):
        outs = issue(i)
    # every stream's work is done before the end mark
    for st in (s_in, s_comp):
        ev = torch.cuda.Event()
        ev.record(st)
        s_out.wait_event(ev)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    total = max_over_ranks(start.elapsed_time(end), world)
    h2d = (M * K + M * N) * 2
    d2h = sum(t.numel() * t.element_size() for t in outs)
    val = (w.flops_fwd + w.flops_bwd) * world * K_steps / (total * 1e-3) / 1e12
    return {"value": round(val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(total / K_steps, 4), "read_back": "+".join(E2E_RESULTS[read_back]),
            "pipelining": "three streams: copies in of step i+1 and out of step i-1 overlap step i; L2 flushed at the "
                          "start of every step's compute (inside the timed interval)"}


def run_other_workloads(peaks, dev):
    """Throughput of the other workloads and of the NF4 round trip (one GPU, device-timed, L2 flushed)."""
    import torch

    from qlora_fine_tuning_blockwise_b200 import inputs as I
    from qlora_fine_tuning_blockwise_b200 import ops

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timeit(fn, reps=10, warm=3):
        for _ in range(warm):
            flush_l2(flush)
            fn()
        tot = 0.0
        for _ in range(reps):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        return tot / reps

    res = {}
    for name in ("mlpdown_4096x11008x4096_r64", "decode_16x8192x28672_r16"):
        w = I.WORKLOADS[name]
        d = I.make_linear_inputs(w)
        layer = ops.QLoRALinear(torch.from_numpy(d["W"]).to(dev), d["A"].to(dev), d["B"].to(dev), d["s"])
        x, dy = d["x"].to(dev), d["dy"].to(dev)
        fwd_ms = timeit(lambda: layer.forward(x))
        entry = {"fwd_ms": round(fwd_ms, 4), "fwd_tflops": round(w.flops_fwd / (fwd_ms * 1e-3) / 1e12, 1),
                 "fwd_gbs": round(w.bytes_fwd / (fwd_ms * 1e-3) / 1e9, 1)}
        fwd_roof = max(w.flops_fwd / (peaks["bf16_tflops"] * 1e12), w.bytes_fwd / (peaks["hbm_gbs"] * 1e9)) * 1e3
        entry["fwd_roofline_frac"] = round(fwd_roof / fwd_ms, 4)
        if w.backward:
            y, su = layer.forward(x)
            bwd_ms = timeit(lambda: layer.backward(dy, x, su=su))
            bwd_roof = max(w.flops_bwd / (peaks["bf16_tflops"] * 1e12), w.bytes_bwd / (peaks["hbm_gbs"] * 1e9)) * 1e3
            entry.update({"bwd_ms": round(bwd_ms, 4), "bwd_tflops": round(w.flops_bwd / (bwd_ms * 1e-3) / 1e12, 1),
                          "bwd_roofline_frac": round(bwd_roof / bwd_ms, 4)})
        res[name] = entry
        del layer, x, dy, d
        torch.cuda.empty_cache()
    # NF4 round trip on the attention-projection weight (4096 x 4096)
    w = I.WORKLOADS[DEFAULT_WORKLOAD]
    W = torch.from_numpy(I.draw_w(I._streams(0), w.N, w.K, w.w_std)).to(dev).reshape(-1)
    n = W.numel()
    q_ms = timeit(lambda: ops.nf4_quantize(W))
    codes, absmax = ops.nf4_quantize(W)
    dq_ms = timeit(lambda: ops.nf4_dequantize(codes, absmax, n, dtype=torch.bfloat16))
    qb = n * 4 + n // 2 + n // 64 * 4
    db = n // 2 + n // 64 * 4 + n * 2
    res["nf4_4096x4096"] = {"quantize_ms": round(q_ms, 4), "quantize_gbs": round(qb / (q_ms * 1e-3) / 1e9, 1),
                            "quantize_hbm_frac": round(qb / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                            "dequantize_bf16_ms": round(dq_ms, 4),
                            "dequantize_gbs": round(db / (dq_ms * 1e-3) / 1e9, 1),
                            "dequantize_hbm_frac": round(db / (dq_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    del W, codes, absmax
    # LoRA merge requantized to NF4 in one pass, on the decode layer's weight (28672 x 8192, r = 16).  Its
    # fixed-order fp32 arithmetic runs on the CUDA cores: 2r + 3 single operations per element (r products,
    # r additions, the dequantizing product, the scaling, the final addition), against one fp32 operation
    # per lane per clock (128 lanes per SM).
    w = I.WORKLOADS["decode_16x8192x28672_r16"]
    d = I.make_linear_inputs(w)
    codes, absmax = ops.nf4_quantize(torch.from_numpy(d["W"]).to(dev).reshape(-1))
    A, B = d["A"].to(dev), d["B"].to(dev)
    c_out, a_out = torch.empty_like(codes), torch.empty_like(absmax)
    m_ms = timeit(lambda: ops.merge_lora_nf4(codes, absmax, A, B, w.s, w.N, w.K, codes_out=c_out, absmax_out=a_out))
    n = w.N * w.K
    mb = 2 * (n // 2 + n // 64 * 4) + (w.r * w.K + w.N * w.r) * 2
    alu_ops = n * (2 * w.r + 3)
    alu_peak = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * peaks.get("sm_max_mhz", 1965.0) * 1e6
    res["merge_nf4_28672x8192_r16"] = {"ms": round(m_ms, 4), "gbs": round(mb / (m_ms * 1e-3) / 1e9, 1),
                                       "hbm_frac": round(mb / (m_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                       "alu_gops": round(alu_ops / (m_ms * 1e-3) / 1e9, 1),
                                       "alu_frac": round(alu_ops / (m_ms * 1e-3) / alu_peak, 4)}
    # Weight-format conversions on the same weight: NVFP4 quantize / dequantize (bf16) and the double
    # quantization of its NF4 block constants.  Kept apart so that a failure here cannot lose the line.
    try:
        Wd = torch.from_numpy(d["W"]).to(dev).reshape(-1)
        nb = absmax.numel()
        fq_ms = timeit(lambda: ops.nvfp4_quantize(Wd))
        fc, fs, fS = ops.nvfp4_quantize(Wd)
        fd_ms = timeit(lambda: ops.nvfp4_dequantize(fc, fs, fS, n, dtype=torch.bfloat16))
        dq_ms = timeit(lambda: ops.nf4_double_quantize(absmax))
        q8, c1, mu = ops.nf4_double_quantize(absmax)
        dd_ms = timeit(lambda: ops.nf4_double_dequantize(q8, c1, mu))
        fqb = 2 * n * 4 + n // 2 + n // 16     # the weight read twice (largest magnitude, then blocks)
        fdb = n // 2 + n // 16 + n * 2
        dqb = 2 * nb * 4 + nb + (nb + 255) // 256 * (4 + 2 * 8)
        ddb = nb + (nb + 255) // 256 * 4 + nb * 4

        def hbm(b, ms):
            return {"ms": round(ms, 4), "gbs": round(b / (ms * 1e-3) / 1e9, 1),
                    "hbm_frac": round(b / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
        res["formats_28672x8192"] = {"nvfp4_quantize": hbm(fqb, fq_ms), "nvfp4_dequantize_bf16": hbm(fdb, fd_ms),
                                     "nf4_double_quantize": hbm(dqb, dq_ms),
                                     "nf4_double_dequantize": hbm(ddb, dd_ms)}
        del Wd, fc, fs, fS, q8, c1, mu
    except Exception as e:  # pragma: no cover - reported, never fatal for the main line
        res["formats_28672x8192"] = {"error": f"{type(e).__name__}: {e}"[:200]}
    del d, codes, absmax, A, B, c_out, a_out
    torch.cuda.empty_cache()
    # The gated-MLP block (x [8192, 8192], F = 28672, r = 64 per layer): gate+up as one stacked QLoRA layer,
    # SwiGLU, down; forward, then backward from the saved activations.  Tens of milliseconds per pass, so its
    # fraction is taken against the sustained bf16 peak.
    try:
        from qlora_fine_tuning_blockwise_b200.mlp import QLoRAGatedMLP
        c = I.make_chain_inputs()
        Ls = c["layers"]

        def on(t):
            return (t if isinstance(t, torch.Tensor) else torch.from_numpy(t)).to(dev).contiguous()
        block = QLoRAGatedMLP(on(Ls["gate"]["W"]), on(Ls["up"]["W"]), on(Ls["down"]["W"]), on(Ls["gate"]["A"]),
                              on(Ls["gate"]["B"]), on(Ls["up"]["A"]), on(Ls["up"]["B"]), on(Ls["down"]["A"]),
                              on(Ls["down"]["B"]), c["s"])
        x, dy = on(c["x"]), on(c["dy"])
        del c, Ls
        torch.cuda.empty_cache()
        f_ms = timeit(lambda: block.forward(x), reps=5)
        _, saved = block.forward(x)
        b_ms = timeit(lambda: block.backward(dy, x, saved), reps=5)
        ff, fb = QLoRAGatedMLP.flops(x.shape[0], block.D, block.F, block.r)
        sus = peaks["bf16_tflops_sustained"] * 1e12
        res[I.CHAIN["name"]] = {"fwd_ms": round(f_ms, 3), "fwd_tflops": round(ff / (f_ms * 1e-3) / 1e12, 1),
                                "fwd_frac_of_sustained": round(ff / (f_ms * 1e-3) / sus, 4),
                                "bwd_ms": round(b_ms, 3), "bwd_tflops": round(fb / (b_ms * 1e-3) / 1e12, 1),
                                "bwd_frac_of_sustained": round(fb / (b_ms * 1e-3) / sus, 4),
                                "step_tflops": round((ff + fb) / ((f_ms + b_ms) * 1e-3) / 1e12, 1)}
        del block, x, dy, saved
        torch.cuda.empty_cache()
    except Exception as e:  # pragma: no cover - reported, never fatal for the main line
        res[I.CHAIN["name"]] = {"error": f"{type(e).__name__}: {e}"[:200]}
    return res


# ------------------------------------------------------------------------------------------ oracle (CPU)


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_step_sample(workload: str, m_sample: int):
    """One oracle step (dequantize + fwd + bwd, fp64) on the first m_sample tokens; returns (seconds, flops)."""
    import numpy as np

    from oracle import linear as L
    from oracle import nf4 as O
    from qlora_fine_tuning_blockwise_b200 import inputs as I

    w = I.WORKLOADS[workload]
    d = I.make_linear_inputs(w, M=m_sample)
    codes, absmax = O.nf4_quantize(d["W"])  # the frozen weight is quantized once, outside the step
    f = lambda t: t.float().numpy().astype(np.float64)
    x, A, B, dy = f(d["x"]), f(d["A"]), f(d["B"]), f(d["dy"])
    t0 = time.perf_counter()
    Wd = L.dequantized_weight(codes, absmax, w.N, w.K)
    L.qlora_forward(x, Wd, A, B, w.s)
    L.qlora_backward(dy, x, Wd, A, B, w.s)
    dt = time.perf_counter() - t0
    Ms, N, K, r = m_sample, w.N, w.K, w.r
    flops = (2 * Ms * N * K + 2 * Ms * K * r + 2 * Ms * N * r) + (2 * Ms * N * K + 2 * Ms * N * r + 2 * Ms * r * K
                                                                 + 2 * r * Ms * K + 2 * N * Ms * r)
    return dt, flops


def cpu_baseline(workload: str, target_s: float = 12.0, max_steps: int = 60) -> dict:
    """The oracle as it stands, on a bounded sample of about `target_s` seconds of host work: a token sub-batch
    when one full step would take longer, else whole steps repeated until the target (at most `max_steps`)."""
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    M = I.WORKLOADS[workload].M
    dt, flops = oracle_step_sample(workload, min(256, M))
    m_sample = int(min(M, max(64, min(256, M) * target_s / max(dt, 1e-3))))
    m_sample -= m_sample % 64 if m_sample > 64 else 0
    if m_sample != min(256, M):
        dt, flops = oracle_step_sample(workload, m_sample)
    steps, tot_t, tot_f = 1, dt, flops
    while tot_t < target_s and steps < max_steps:
        dt, flops = oracle_step_sample(workload, m_sample)
        tot_t += dt
        tot_f += flops
        steps += 1
    return {"value": round(tot_f / tot_t / 1e12, 5), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{workload}, first {m_sample} of its {M} tokens, {steps} step(s) of dequantize + fwd + bwd "
                      f"in fp64 (numpy), {tot_t:.1f} s timed", "seconds": round(tot_t, 3)}


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, each step a bounded sub-batch of the workload."""
    m_sample = args.ref_tokens
    for _ in range(args.warmup):
        oracle_step_sample(args.workload, m_sample)
    tot_t, tot_f = 0.0, 0
    for _ in range(args.steps):
        dt, fl = oracle_step_sample(args.workload, m_sample)
        tot_t += dt
        tot_f += fl
    val = tot_f / tot_t / 1e12
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    out = {
        "impl": "reference", "metric": METRIC, "value": round(val, 5), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "r": w.r, "s": w.s,
                   "sampled_tokens_per_step": m_sample, "parallelism": f"dp{args.gpus}"},
        "cpu_baseline": {"value": round(val, 5), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"first {m_sample} of {w.M} tokens per step, dequantize + fwd + bwd, fp64 numpy"},
        "e2e": {"value": round(val, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--only-main", action="store_true", help="skip the other workloads and the CPU baseline")
    ap.add_argument("--ref-tokens", type=int, default=256, help="tokens per oracle step (reference arm)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return

    peaks = load_peaks()
    rank, world, local = dist_setup(args.gpus)
    out, ctx = run_ours(args, rank, world, local, peaks)
    out["e2e"] = run_e2e(ctx, args, world, "grads")
    full = run_e2e(ctx, args, world, "all")
    out["e2e"]["all_outputs"] = {k: full[k] for k in ("value", "ms_per_step", "d2h_bytes_per_step", "read_back")}
    if rank == 0 and world == 1:
        import torch
        if not args.only_main:
            out["workloads"] = run_other_workloads(peaks, ctx[5])
            torch.cuda.synchronize()
        out["cpu_baseline"] = cpu_baseline(args.workload)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
