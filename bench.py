#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 layers (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME] [--only-main]

The default workload is the largest: the gated-MLP block ``mlpchain_8192x8192x28672_r64`` (8192 tokens of width
8192; gate and up projections to F = 28672 and the down projection back, each an NF4 layer with its own rank-64
LoRA pair, SwiGLU between).  One step = one training step of the block over one batch of synthetic tokens:
forward (s*x*A^T; the stacked gate/up GEMM with the SwiGLU in its epilogue; the down layer) and backward (the
down layer's dX GEMM with dSwiGLU in its epilogue, its dA, dB; the gate/up dX GEMM, dA, dB).  A linear workload
name (e.g. ``attn_2048x4096x4096_r16``) benchmarks a single layer instead.  With N > 1 ranks each rank runs its
own batch (data parallel, weak scaling) and the adapter gradients are summed over ranks with NCCL.  NF4 weights
are quantized once before timing (they are frozen), as in fine-tuning.

Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the launching stream; the L2 is flushed
(256 MiB written, then read back so that L2 holds clean lines) before every step outside the timed interval;
barrier + synchronize on both sides of the timed loop; the result is the max over ranks.  rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference that exists for these layers) on a bounded sample
of the same workload, on the host cores, rank 0 only.
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
CHAIN_WORKLOAD = "mlpchain_8192x8192x28672_r64"
DEFAULT_WORKLOAD = CHAIN_WORKLOAD
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
# the bounded sample the CPU oracle runs per step for the block: its first CHAIN_SAMPLE_TOKENS tokens (the
# reference arm's --ref-tokens) and the first F / CHAIN_SAMPLE_F_DIV of its intermediate features
CHAIN_SAMPLE_TOKENS = 64
CHAIN_SAMPLE_F_DIV = 8


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
# whose counters are recorded under profiles/ are built from these and nothing else.  The format conversions'
# kernels (formats.cu) are a separate translation unit; their per-element arithmetic (formats.cuh) is shared
# with the FP4 path's activation quantizer.
LAYER_SOURCES = ("elementwise.cuh", "formats.cuh", "fp4_gemm.cuh", "nf4_table.cuh", "ptx.cuh", "qlora.cu",
                 "swiglu.cuh", "umma_gemm.cuh")


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


def load_traffic(workload: str) -> dict:
    """ncu DRAM bytes per launch of each fused kernel of ``workload``, recorded under profiles/; valid only for
    the kernel source they were taken on ({} otherwise)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except Exception:
        return {}
    if t.get("source_sha") != kernel_source_sha():
        return {}
    return dict(t.get("workloads", {}).get(workload, {}))


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or "unknown"


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


def flush_l2(buf):
    """Evict the workload from L2: write a 256 MiB buffer, then read it back.  The read leaves L2 holding clean
    lines of the flush buffer, so the timed kernels do not pay for writing the flush's dirty lines back to HBM
    (on a B200 that write-back cost a 30 us, 132 MB streaming kernel about 8 us)."""
    import torch
    buf.zero_()
    buf.view(torch.int64).sum()  # one read pass, no cast


# ------------------------------------------------------------------------------------------ work per workload


CHAIN_TOKENS = [None]  # --tokens: a smaller token batch of the block (for profiler captures); None = 8192


def chain_dims():
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    c = I.CHAIN
    return CHAIN_TOKENS[0] or c["M"], c["D"], c["F"], c["r"]


def chain_flops(M: int, D: int, F: int, r: int) -> tuple[int, int]:
    """Algorithmic (fwd, bwd) FLOPs of the gated-MLP block: three rank-r QLoRA layers (gate, up: D -> F; down:
    F -> D), each 2MNK for the base product plus its LoRA products; SwiGLU and dequantization not counted."""
    def fwd(N, K):
        return 2 * M * N * K + 2 * M * K * r + 2 * M * N * r

    def bwd(N, K):
        return 2 * M * N * K + 2 * M * N * r + 2 * M * r * K + 2 * r * M * K + 2 * N * M * r
    return 2 * fwd(F, D) + fwd(D, F), 2 * bwd(F, D) + bwd(D, F)


def chain_bytes(M: int, D: int, F: int, r: int) -> tuple[int, int]:
    """Algorithmic HBM bytes (fwd, bwd): every NF4 weight once (0.5625 B per element), every activation and
    gradient read or written once (bf16), adapters once, fp32 adapter gradients written once."""
    w = 3 * F * D * 9 // 16
    lora = 2 * (2 * r * D + 2 * F * r) + (2 * r * F + 2 * D * r)
    fwd = w + lora + 2 * M * D + 2 * M * 2 * F + 2 * M * F + 2 * M * D  # x; gu and h written; y written
    # dY, h, gu read; dgu written and read; x read; dX written; fp32 dA/dB of the three layers written
    bwd = (w + lora + 2 * M * D + 2 * M * F + 2 * M * 2 * F + 2 * 2 * M * 2 * F + 2 * M * D + 2 * M * D
           + 2 * lora)
    return fwd, bwd


def chain_kernel_flops(M: int, D: int, F: int, r: int) -> dict:
    """Algorithmic FLOPs of the four fused GEMM launches of a block step (what each one computes)."""
    return {
        # [x | s u] . [deq(W_gu) | B]^T over the stacked gate/up rows: base 2 M 2F D, LoRA 2 M F r per half
        "gate_up_fwd": 2 * M * 2 * F * D + 2 * 2 * M * F * r,
        "down_fwd": 2 * M * D * F + 2 * M * D * r,
        # dh = dY deq(W_down) + v A_down (then dSwiGLU in the epilogue)
        "down_dx": 2 * M * D * F + 2 * M * r * F,
        # dX = [dg | dup] deq(W_gu) + [v_g | v_u] [A_g; A_u]
        "gate_up_dx": 2 * M * 2 * F * D + 2 * M * 2 * r * D,
    }


# ------------------------------------------------------------------------------------------ our arm: the block


def build_chain(dev, rank: int):
    import torch

    from qlora_fine_tuning_blockwise_b200 import inputs as I
    from qlora_fine_tuning_blockwise_b200.mlp import QLoRAGatedMLP

    c = I.make_chain_inputs(M=chain_dims()[0])
    Ls = c["layers"]

    def on(t):
        return (t if isinstance(t, torch.Tensor) else torch.from_numpy(t)).to(dev).contiguous()
    block = QLoRAGatedMLP(on(Ls["gate"]["W"]), on(Ls["up"]["W"]), on(Ls["down"]["W"]), on(Ls["gate"]["A"]),
                          on(Ls["gate"]["B"]), on(Ls["up"]["A"]), on(Ls["up"]["B"]), on(Ls["down"]["A"]),
                          on(Ls["down"]["B"]), c["s"])
    x_h, dy_h = c["x"], c["dy"]
    if rank:  # every rank its own tokens (data parallel); the frozen weights and the adapters are replicas
        x_h = I.draw_x(I._streams(1000 + rank), c["M"], c["D"])
        dy_h = I.draw_dy(c["M"], c["D"], 2000 + rank)
    del c, Ls
    torch.cuda.empty_cache()
    return block, x_h, dy_h


def chain_grads_list(grads: dict) -> list:
    """The block's adapter gradients as whole tensors (the stacked gate/up dA and dB, and the down pair)."""
    return [grads["gate"][0]._base if grads["gate"][0]._base is not None else grads["gate"][0],
            grads["gate"][1]._base if grads["gate"][1]._base is not None else grads["gate"][1],
            grads["down"][0], grads["down"][1]]


def run_ours_chain(args, rank, world, local, peaks):
    import torch
    import torch.distributed as dist

    from qlora_fine_tuning_blockwise_b200 import build as qbuild
    from qlora_fine_tuning_blockwise_b200 import ops
    from qlora_fine_tuning_blockwise_b200.parallel import allreduce_adapter_grads

    qbuild.build()
    dev = torch.device("cuda", local)
    block, x_h, dy_h = build_chain(dev, rank)
    x, dy = x_h.to(dev), dy_h.to(dev)
    M, D, F, r = chain_dims()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    tags = ("gate_up_fwd", "down_fwd", "down_dx", "gate_up_dx")
    slot = {"gate_up_fwd": 0, "down_fwd": 0, "down_dx": 1, "gate_up_dx": 1}
    cur = {}

    def hook(tag):
        ev = cur.get(tag)
        if ev is not None:
            ops.set_profile_events(slot[tag], ev[0], ev[1])

    block.on_kernel = hook

    def step():
        y, saved = block.forward(x)
        dx, grads = block.backward(dy, x, saved)
        if world > 1:
            allreduce_adapter_grads(chain_grads_list(grads))
        return y, dx, grads

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 + 2 * len(tags))] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = ops.launch_count()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush_l2(flush)
            e = ev[i]
            cur.clear()
            cur.update({t: (e[2 + 2 * j], e[3 + 2 * j]) for j, t in enumerate(tags)})
            e[0].record(stream)
            step()
            e[1].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    cur.clear()
    block.on_kernel = None
    ops.set_profile_events(0, None, None)
    ops.set_profile_events(1, None, None)
    launches = ops.launch_count() - launches0
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world)
    ms_per_step = total_ms / K
    ff, fb = chain_flops(M, D, F, r)
    value = (ff + fb) * world * K / (total_ms * 1e-3) / 1e12

    kflops = chain_kernel_flops(M, D, F, r)
    kern = {}
    for j, t in enumerate(tags):
        ms = sum(e[2 + 2 * j].elapsed_time(e[3 + 2 * j]) for e in ev) / K
        kern[t] = {"ms": ms, "flops": kflops[t], "tflops": kflops[t] / (ms * 1e-3) / 1e12}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    ach = kern[dom]["tflops"]
    traffic = load_traffic(CHAIN_WORKLOAD).get(dom)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4),
                "peak_source": peaks["source"] + " bf16 burst", "traffic": traffic,
                "kernel_ms": round(kern[dom]["ms"], 4),
                "frac_of_sustained": round(ach / peaks["bf16_tflops_sustained"], 4),
                "kernels": {k: {"ms": round(v["ms"], 4), "tflops": round(v["tflops"], 1),
                                "frac": round(v["tflops"] / peaks["bf16_tflops"], 4)} for k, v in kern.items()}}
    bf, bb = chain_bytes(M, D, F, r)
    step_roof_ms = max((ff + fb) / (peaks["bf16_tflops"] * 1e12), (bf + bb) / (peaks["hbm_gbs"] * 1e9)) * 1e3
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": CHAIN_WORKLOAD, "M": M, "D": D, "F": F, "r": r, "s": 2.0, "tokens_per_rank": M,
                   "global_tokens": M * world, "parallelism": f"dp{world}",
                   "layers": "gate+up (stacked, SwiGLU in the epilogue) and down, NF4 block 64, one LoRA pair each",
                   "l2": "flushed before every timed step (256 MiB written, then read back; outside the timed interval); inputs "
                         "(134 MB activations, 396 MB of NF4 weights) exceed the 126 MB L2"},
        "roofline": roofline,
        "step_roofline_frac": round(step_roof_ms / ms_per_step, 4),
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    return out, (block, x_h, dy_h, dev)


def run_e2e_chain(ctx, args, world):
    """Same metric through the public API with host buffers: every step copies its x and dY in from pinned host
    memory and reads its result -- the adapter gradients of the three layers -- back to pinned host memory.  Steps
    are pipelined over three streams: the host-to-device copies of step i + 1 and the device-to-host copies of
    step i - 1 overlap step i's compute, with double-buffered device inputs; a step's forward waits for its x
    only, its backward for its dY (whose copy overlaps the forward) and for the gradients of step i - 1 to have
    left the device.  The L2 flush runs at the start of every step's compute,
    inside the timed interval.  Time = device time from the first copy in to the last copy out, max over ranks."""
    import torch
    import torch.distributed as dist

    from qlora_fine_tuning_blockwise_b200.parallel import allreduce_adapter_grads

    block, x_h0, dy_h0, dev = ctx
    x_h, dy_h = x_h0.pin_memory(), dy_h0.pin_memory()
    M, D, F, r = chain_dims()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    slots = [dict(x=torch.empty(M, D, dtype=torch.bfloat16, device=dev),
                  dy=torch.empty(M, D, dtype=torch.bfloat16, device=dev),
                  x_ready=torch.cuda.Event(), dy_ready=torch.cuda.Event(), consumed=torch.cuda.Event())
             for _ in range(2)]
    host = {}
    computed, out_done = torch.cuda.Event(), torch.cuda.Event()
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    state = {"out_pending": False}

    def issue(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(sl["consumed"])  # step i - 2 has finished reading this slot's inputs
            sl["x"].copy_(x_h, non_blocking=True)
            sl["x_ready"].record(s_in)
            sl["dy"].copy_(dy_h, non_blocking=True)
            sl["dy_ready"].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(sl["x_ready"])
            flush_l2(flush)
            y, saved = block.forward(sl["x"])
            s_comp.wait_event(sl["dy_ready"])
            if state["out_pending"]:
                s_comp.wait_event(out_done)  # the previous step's gradients have been read back
            dx, grads = block.backward(sl["dy"], sl["x"], saved)
            outs = chain_grads_list(grads)
            if world > 1:
                allreduce_adapter_grads(outs)
            sl["consumed"].record(s_comp)
            computed.record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed)
            for j, t in enumerate(outs):
                h = host.get(j)
                if h is None:
                    h = host[j] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                h.copy_(t, non_blocking=True)
            out_done.record(s_out)
        state["out_pending"] = True
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
    for st in (s_in, s_comp):
        ev = torch.cuda.Event()
        ev.record(st)
        s_out.wait_event(ev)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    total = max_over_ranks(start.elapsed_time(end), world)
    h2d = 2 * M * D * 2
    d2h = sum(t.numel() * t.element_size() for t in outs)
    ff, fb = chain_flops(M, D, F, r)
    val = (ff + fb) * world * K_steps / (total * 1e-3) / 1e12
    return {"value": round(val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(total / K_steps, 4), "read_back": "dA+dB of gate/up (stacked) and down",
            "pipelining": "three streams: copies in of step i+1 and out of step i-1 overlap step i, and a step's dY "
                          "copy overlaps its forward; L2 flushed at the start of every step's compute (inside the "
                          "timed interval)"}


# ------------------------------------------------------------------------------------------ our arm: one layer


def run_ours_linear(args, rank, world, local, peaks):
    import torch
    import torch.distributed as dist

    from qlora_fine_tuning_blockwise_b200 import build as qbuild
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    from qlora_fine_tuning_blockwise_b200 import ops
    from qlora_fine_tuning_blockwise_b200.parallel import allreduce_adapter_grads

    qbuild.build()
    w = I.WORKLOADS[args.workload]
    d = I.make_linear_inputs(w, seed=0)
    if rank:
        d["x"] = I.draw_x(I._streams(1000 + rank), w.M, w.K, w.x_kind)
        d["dy"] = I.draw_dy(w.M, w.N, 2000 + rank)
    dev = torch.device("cuda", local)
    if args.fp4:  # the NVFP4 form on the block-scaled FP4 tensor core: forward only
        import dataclasses
        w = dataclasses.replace(w, backward=False)
        layer = ops.FP4Linear(torch.from_numpy(d["W"]).to(dev), d["A"].to(dev), d["B"].to(dev), d["s"])
    else:
        layer = ops.QLoRALinear(torch.from_numpy(d["W"]).to(dev), d["A"].to(dev), d["B"].to(dev), d["s"])
    x = d["x"].to(dev)
    dy = d["dy"].to(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        y, su = layer.forward(x)
        if not w.backward:
            return y, None, None, None
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
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world)
    ms_per_step = total_ms / K
    flops_step = w.flops_fwd + (w.flops_bwd if w.backward else 0)
    bytes_step = w.bytes_fwd + (w.bytes_bwd if w.backward else 0)
    value = flops_step * world * K / (total_ms * 1e-3) / 1e12
    M, N, Kd, r = w.M, w.N, w.K, w.r
    kern = {"fused_fwd": {"ms": sum(e[2].elapsed_time(e[3]) for e in ev) / K, "flops": 2 * M * N * Kd + 2 * M * N * r}}
    if w.backward:
        kern["fused_dx"] = {"ms": sum(e[4].elapsed_time(e[5]) for e in ev) / K, "flops": 2 * M * N * Kd + 2 * M * Kd * r}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    traffic = load_traffic(w.name).get(dom)
    if args.fp4:
        ach = kern[dom]["flops"] / (kern[dom]["ms"] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "fp4_gemm", "achieved": round(ach, 1), "peak": 4 * peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(ach / (4 * peaks["bf16_tflops"]), 4),
                    "peak_source": peaks["source"] + " bf16 burst x 4 (nominal dense FP4 / bf16 ratio)",
                    "traffic": load_traffic(w.name + "_fp4").get("fp4_gemm"), "kernel_ms": round(kern[dom]["ms"], 4)}
    elif w.backward:
        ach = kern[dom]["flops"] / (kern[dom]["ms"] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 1), "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4),
                    "peak_source": peaks["source"] + " bf16 burst", "traffic": traffic,
                    "kernel_ms": round(kern[dom]["ms"], 4)}
    else:  # token-light forward: bound by streaming the weight
        ach = w.bytes_fwd / (kern[dom]["ms"] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                    "peak_source": peaks["source"] + " HBM copy", "traffic": traffic,
                    "kernel_ms": round(kern[dom]["ms"], 4)}
    step_roof_ms = max(flops_step / (peaks["bf16_tflops"] * 1e12), bytes_step / (peaks["hbm_gbs"] * 1e9)) * 1e3
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1" if args.fp4 else "bf16", "data": "synthetic",
        "config": {"workload": w.name + ("_fp4" if args.fp4 else ""), "M": M, "N": N, "K": Kd, "r": r, "s": w.s,
                   "tokens_per_rank": M,
                   "global_tokens": M * world, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (256 MiB written, then read back; outside the timed interval)"},
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


def run_e2e_fp4(ctx, args, world):
    """The NVFP4 forward through its public call with host buffers: x copied in, y read back, pipelined as the
    other end-to-end measurements."""
    import torch

    layer, _x, _dy, d, w, dev = ctx
    x_h = d["x"].pin_memory()
    M, N = w.M, w.N
    slots = [dict(x=torch.empty_like(d["x"], device=dev), y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                  h=torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True), ready=torch.cuda.Event(),
                  done=torch.cuda.Event(), out=torch.cuda.Event()) for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def issue(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(sl["done"])
            sl["x"].copy_(x_h, non_blocking=True)
            sl["ready"].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(sl["ready"])
            if i >= 2:
                s_comp.wait_event(sl["out"])
            layer.forward(sl["x"], y=sl["y"])
            sl["done"].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sl["done"])
            sl["h"].copy_(sl["y"], non_blocking=True)
            sl["out"].record(s_out)

    for i in range(max(args.warmup, 3)):
        issue(i)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(args.steps):
        issue(i)
    for st in (s_in, s_comp):
        ev = torch.cuda.Event()
        ev.record(st)
        s_out.wait_event(ev)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    total = max_over_ranks(start.elapsed_time(end), world)
    val = w.flops_fwd * world * args.steps / (total * 1e-3) / 1e12
    return {"value": round(val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(M * w.K * 2),
            "d2h_bytes_per_step": int(M * N * 2), "ms_per_step": round(total / args.steps, 4), "read_back": "y"}


def run_e2e_linear(ctx, args, world, read_back: str = "grads"):
    """One layer through the public API with host buffers: every step copies its x and dY in from pinned host
    memory and its result out to pinned host memory (``E2E_RESULTS[read_back]``), pipelined over three streams
    with double-buffered device inputs and outputs, as for the block."""
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
    names_for = E2E_RESULTS[read_back] if w.backward else ("y",)

    def issue(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(sl["computed"])  # step i - 2 has finished reading this slot's inputs
            sl["x"].copy_(x_h, non_blocking=True)
            if w.backward:
                sl["dy"].copy_(dy_h, non_blocking=True)
            sl["in_ready"].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(sl["in_ready"])
            if i >= 2:
                s_comp.wait_event(sl["out_done"])  # step i - 2's outputs have left this slot
            flush_l2(flush)
            ops.qlora_linear_fwd(sl["x"], layer.codes, layer.absmax, layer.A, layer.B, layer.s, N, K,
                                 workspace=bufs["ws_f"], y=sl["y"], su=sl["su"])
            if w.backward:
                ops.qlora_linear_bwd(sl["dy"], sl["x"], layer.codes, layer.absmax, layer.A, layer.B, layer.s, N, K,
                                     su=sl["su"], workspace=bufs["ws_b"], dx=sl["dx"], dA=sl["dA"], dB=sl["dB"])
                if world > 1:
                    allreduce_adapter_grads([sl["dA"], sl["dB"]])
            sl["computed"].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sl["computed"])
            names = [nm for nm in names_for if sl[nm] is not None] or ["dx"]  # r = 0: no gradients
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
    for st in (s_in, s_comp):
        ev = torch.cuda.Event()
        ev.record(st)
        s_out.wait_event(ev)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    total = max_over_ranks(start.elapsed_time(end), world)
    h2d = (M * K + (M * N if w.backward else 0)) * 2
    d2h = sum(t.numel() * t.element_size() for t in outs)
    val = (w.flops_fwd + (w.flops_bwd if w.backward else 0)) * world * K_steps / (total * 1e-3) / 1e12
    return {"value": round(val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(total / K_steps, 4), "read_back": "+".join(names_for),
            "pipelining": "three streams: copies in of step i+1 and out of step i-1 overlap step i; L2 flushed at the "
                          "start of every step's compute (inside the timed interval)"}


# ------------------------------------------------------------------------------------------ other workloads


def run_other_workloads(peaks, dev):
    """Each single-layer workload (attention projection, MLP down projection, decode) with its own roofline
    fractions, and the one-time conversions (NF4 round trip, LoRA merge, weight formats).  One GPU, device-timed,
    L2 flushed before every timed call."""
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

    def kernel_ms(fn, which, reps=10, warm=3):
        """Average duration of the fused GEMM launch `which` (0 forward, 1 dX) inside fn, by the library's
        profiling events."""
        for _ in range(warm):
            flush_l2(flush)
            fn()
        tot = 0.0
        for _ in range(reps):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ops.set_profile_events(which, a, b)
            fn()
            b.synchronize()
            tot += a.elapsed_time(b)
        ops.set_profile_events(which, None, None)
        return tot / reps

    res = {}
    for name in ("attn_2048x4096x4096_r16", "mlpdown_4096x11008x4096_r64", "decode_16x8192x28672_r16"):
        try:
            w = I.WORKLOADS[name]
            d = I.make_linear_inputs(w)
            layer = ops.QLoRALinear(torch.from_numpy(d["W"]).to(dev), d["A"].to(dev), d["B"].to(dev), d["s"])
            x, dy = d["x"].to(dev), d["dy"].to(dev)
            M, N, K, r = w.M, w.N, w.K, w.r
            fwd_ms = timeit(lambda: layer.forward(x))
            kf_ms = kernel_ms(lambda: layer.forward(x), 0)
            fwd_roof = max(w.flops_fwd / (peaks["bf16_tflops"] * 1e12), w.bytes_fwd / (peaks["hbm_gbs"] * 1e9)) * 1e3
            entry = {"fwd_ms": round(fwd_ms, 4), "fwd_tflops": round(w.flops_fwd / (fwd_ms * 1e-3) / 1e12, 1),
                     "fwd_gbs": round(w.bytes_fwd / (fwd_ms * 1e-3) / 1e9, 1),
                     "fwd_roofline_frac": round(fwd_roof / fwd_ms, 4), "fused_fwd_ms": round(kf_ms, 4)}
            kfl = 2 * M * N * K + 2 * M * N * r
            if w.backward:
                entry["fused_fwd_frac"] = round(kfl / (kf_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)
                y, su = layer.forward(x)
                bwd_ms = timeit(lambda: layer.backward(dy, x, su=su))
                kd_ms = kernel_ms(lambda: layer.backward(dy, x, su=su), 1)
                bwd_roof = max(w.flops_bwd / (peaks["bf16_tflops"] * 1e12),
                               w.bytes_bwd / (peaks["hbm_gbs"] * 1e9)) * 1e3
                kdl = 2 * M * N * K + 2 * M * K * r
                entry.update({"bwd_ms": round(bwd_ms, 4), "bwd_tflops": round(w.flops_bwd / (bwd_ms * 1e-3) / 1e12, 1),
                              "bwd_roofline_frac": round(bwd_roof / bwd_ms, 4), "fused_dx_ms": round(kd_ms, 4),
                              "fused_dx_frac": round(kdl / (kd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                              "step_ms": round(fwd_ms + bwd_ms, 4),
                              "step_tflops": round((w.flops_fwd + w.flops_bwd) / ((fwd_ms + bwd_ms) * 1e-3) / 1e12, 1)})
            else:
                entry["fused_fwd_hbm_frac"] = round(w.bytes_fwd / (kf_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
            entry["traffic"] = load_traffic(name) or None
            res[name] = entry
            del layer, x, dy, d
            torch.cuda.empty_cache()
        except Exception as e:  # pragma: no cover - reported, never fatal for the main line
            res[name] = {"error": f"{type(e).__name__}: {e}"[:200]}
    # The decode layer on double-quantized NF4 constants (8-bit E4M3 codes, an fp32 scale per 256 and an offset
    # instead of fp32 absmax): the fused GEMM reads the compressed constants, so its algorithmic bytes drop by
    # 11 MB; the fraction is taken against those bytes.
    try:
        w = I.WORKLOADS["decode_16x8192x28672_r16"]
        d = I.make_linear_inputs(w)
        wt = ops.Weight.nf4_dq(torch.from_numpy(d["W"]).to(dev))
        A, B, x = d["A"].to(dev), d["B"].to(dev), d["x"].to(dev)
        M, N, K, r = w.M, w.N, w.K, w.r
        f_ms = timeit(lambda: ops.linear_fwd_w(x, wt, A, B, w.s))
        k_ms = kernel_ms(lambda: ops.linear_fwd_w(x, wt, A, B, w.s), 0)
        nb = N * K // 64
        dq_bytes = N * K // 2 + nb + (nb + 255) // 256 * 4 + 4 + 2 * M * K + 2 * M * N + 2 * r * K + 2 * N * r
        res["decode_16x8192x28672_r16_nf4dq"] = {
            "fwd_ms": round(f_ms, 4), "fwd_gbs": round(dq_bytes / (f_ms * 1e-3) / 1e9, 1),
            "fwd_roofline_frac": round(dq_bytes / (f_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "fused_fwd_ms": round(k_ms, 4),
            "fused_fwd_hbm_frac": round(dq_bytes / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "algorithmic_bytes": int(dq_bytes), "nf4_algorithmic_bytes": int(w.bytes_fwd)}
        del wt, A, B, x, d
        torch.cuda.empty_cache()
    except Exception as e:  # pragma: no cover - reported, never fatal for the main line
        res["decode_16x8192x28672_r16_nf4dq"] = {"error": f"{type(e).__name__}: {e}"[:200]}
    # The NVFP4 form of the layer on the block-scaled FP4 tensor core: the layer forward (activation quantization,
    # s x A^T, the FP4 GEMM) and the FP4 GEMM alone.  Its peak is the measured bf16 peak times 4, the ratio of
    # the nominal dense FP4 and bf16 tensor rates (9 and 2.25 PFLOP/s).
    fp4_peak = 4.0 * peaks["bf16_tflops"]
    for name in ("attn_2048x4096x4096_r16", "mlpdown_4096x11008x4096_r64", "decode_16x8192x28672_r16"):
        try:
            w = I.WORKLOADS[name]
            d = I.make_linear_inputs(w)
            layer = ops.FP4Linear(torch.from_numpy(d["W"]).to(dev), d["A"].to(dev), d["B"].to(dev), d["s"])
            x = d["x"].to(dev)
            M, N, K, r = w.M, w.N, w.K, w.r
            f_ms = timeit(lambda: layer.forward(x))
            k_ms = kernel_ms(lambda: layer.forward(x), 0)
            kfl = 2 * M * N * K + 2 * M * N * r
            wbytes = N * K // 2 + N * K // 16 + 2 * M * K + 2 * M * N  # fp4 weight + its scales, x in, y out
            res["fp4_" + name] = {
                "fwd_ms": round(f_ms, 4), "fwd_tflops": round(w.flops_fwd / (f_ms * 1e-3) / 1e12, 1),
                "fp4_gemm_ms": round(k_ms, 4), "fp4_gemm_tflops": round(kfl / (k_ms * 1e-3) / 1e12, 1),
                "fp4_gemm_frac_of_fp4_peak": round(kfl / (k_ms * 1e-3) / 1e12 / fp4_peak, 4),
                "fp4_gemm_gbs": round(wbytes / (k_ms * 1e-3) / 1e9, 1),
                "fp4_peak_tflops": fp4_peak, "peak_note": "4 x measured bf16 (nominal dense FP4 / bf16 ratio)"}
            del layer, x, d
            torch.cuda.empty_cache()
        except Exception as e:  # pragma: no cover - reported, never fatal for the main line
            res["fp4_" + name] = {"error": f"{type(e).__name__}: {e}"[:200]}
    # NF4 round trip on the attention-projection weight (4096 x 4096)
    w = I.WORKLOADS["attn_2048x4096x4096_r16"]
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


class ChainSample:
    """The block's bounded oracle sample: its first m tokens and first f intermediate features, quantized to
    NF4 by the oracle once (the frozen weights), outside any timed step."""

    def __init__(self, m: int, f: int):
        import numpy as np

        from oracle import nf4 as O
        from qlora_fine_tuning_blockwise_b200 import inputs as I

        c = I.make_chain_sample(m, f)
        self.m, self.f, self.D, self.r, self.s = m, f, c["D"], c["r"], c["s"]
        fl = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
        self.x, self.dy = fl(c["x"]), fl(c["dy"])
        self.layers = {}
        for name, L in c["layers"].items():
            codes, absmax = O.nf4_quantize(L["W"])
            self.layers[name] = dict(codes=codes, absmax=absmax, N=L["N"], K=L["K"], A=fl(L["A"]), B=fl(L["B"]))

    def flops(self) -> int:
        ff, fb = chain_flops(self.m, self.D, self.f, self.r)
        return ff + fb

    def step(self) -> float:
        """One oracle step (dequantize the three weights, then the block's forward and backward in fp64);
        returns the seconds it took."""
        from oracle import linear as L
        t0 = time.perf_counter()
        p = {}
        for name, d in self.layers.items():
            p[name] = (L.dequantized_weight(d["codes"], d["absmax"], d["N"], d["K"]), d["A"], d["B"], self.s)
        y, g, u, h = L.mlp_chain_forward(self.x, p["gate"], p["up"], p["down"])
        L.mlp_chain_backward(self.dy, self.x, p["gate"], p["up"], p["down"], (g, u, h))
        return time.perf_counter() - t0

    def describe(self) -> str:
        return (f"{CHAIN_WORKLOAD}: its first {self.m} of 8192 tokens and first {self.f} of 28672 intermediate "
                f"features (exact slices of the full draws); per step the three weight slices are dequantized and "
                f"the block's forward and backward run in fp64 (numpy)")


def oracle_linear_step_sample(workload: str, m_sample: int):
    """One oracle step of a single layer (dequantize + fwd + bwd, fp64) on its first m_sample tokens; returns
    (seconds, flops)."""
    import numpy as np

    from oracle import linear as L
    from oracle import nf4 as O
    from qlora_fine_tuning_blockwise_b200 import inputs as I

    w = I.WORKLOADS[workload]
    d = I.make_linear_inputs(w, M=m_sample)
    codes, absmax = O.nf4_quantize(d["W"])  # the frozen weight is quantized once, outside the step
    f = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    x, A, B, dy = f(d["x"]), f(d["A"]), f(d["B"]), f(d["dy"])
    t0 = time.perf_counter()
    Wd = L.dequantized_weight(codes, absmax, w.N, w.K)
    L.qlora_forward(x, Wd, A, B, w.s)
    flops = 2 * m_sample * w.N * w.K + 2 * m_sample * w.K * w.r + 2 * m_sample * w.N * w.r
    if w.backward:
        L.qlora_backward(dy, x, Wd, A, B, w.s)
        Ms, N, K, r = m_sample, w.N, w.K, w.r
        flops += 2 * Ms * N * K + 2 * Ms * N * r + 2 * Ms * r * K + 2 * r * Ms * K + 2 * N * Ms * r
    return time.perf_counter() - t0, flops


def timed_steps(step, flops: int, target_s: float, max_steps: int = 60):
    steps, tot_t = 0, 0.0
    while (tot_t < target_s or steps == 0) and steps < max_steps:
        tot_t += step()
        steps += 1
    return steps, tot_t, steps * flops / tot_t / 1e12


def cpu_baseline(workload: str, target_s: float = 10.0, one_core_s: float = 5.0) -> dict:
    """The oracle as it stands, on a bounded sample of the workload, timed on the host cores: all cores for
    about ``target_s`` seconds, then one core (BLAS limited to one thread) for about ``one_core_s``."""
    from threadpoolctl import threadpool_limits
    if workload == CHAIN_WORKLOAD:
        smp = ChainSample(CHAIN_SAMPLE_TOKENS, 28672 // CHAIN_SAMPLE_F_DIV)
        step, flops, desc = smp.step, smp.flops(), smp.describe()
    else:
        from qlora_fine_tuning_blockwise_b200 import inputs as I
        M = I.WORKLOADS[workload].M
        m = min(256, M)
        flops = oracle_linear_step_sample(workload, m)[1]
        step = lambda: oracle_linear_step_sample(workload, m)[0]  # noqa: E731
        desc = f"{workload}: its first {m} of {M} tokens; dequantize + fwd (+ bwd) in fp64 (numpy) per step"
    steps, tot, val = timed_steps(step, flops, target_s)
    with threadpool_limits(limits=1, user_api="blas"):
        steps1, tot1, val1 = timed_steps(step, flops, one_core_s)
    return {"value": round(val, 5), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{desc}; {steps} step(s), {tot:.1f} s timed", "seconds": round(tot, 3),
            "cpu_model": cpu_model(), "one_core": {"value": round(val1, 6), "unit": "TFLOP/s", "cores": 1,
                                                   "steps": steps1, "seconds": round(tot1, 3)}}


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, each step a bounded sample of the workload."""
    if args.workload == CHAIN_WORKLOAD:
        smp = ChainSample(args.ref_tokens, 28672 // CHAIN_SAMPLE_F_DIV)
        step, flops, desc = smp.step, smp.flops(), smp.describe()
        config = {"workload": CHAIN_WORKLOAD, "M": 8192, "D": 8192, "F": 28672, "r": 64, "s": 2.0,
                  "sampled_tokens_per_step": args.ref_tokens, "sampled_features_per_step": smp.f,
                  "parallelism": f"dp{args.gpus}"}
    else:
        from qlora_fine_tuning_blockwise_b200 import inputs as I
        w = I.WORKLOADS[args.workload]
        m = args.ref_tokens
        flops = oracle_linear_step_sample(args.workload, m)[1]
        step = lambda: oracle_linear_step_sample(args.workload, m)[0]  # noqa: E731
        desc = f"{w.name}: its first {m} of {w.M} tokens per step; dequantize + fwd (+ bwd), fp64 numpy"
        config = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "r": w.r, "s": w.s,
                  "sampled_tokens_per_step": m, "parallelism": f"dp{args.gpus}"}
    for _ in range(args.warmup):
        step()
    tot_t = 0.0
    for _ in range(args.steps):
        tot_t += step()
    val = flops * args.steps / tot_t / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 5), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": round(val, 5), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": round(val, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--only-main", action="store_true", help="skip the other workloads and the CPU baseline")
    ap.add_argument("--ref-tokens", type=int, default=CHAIN_SAMPLE_TOKENS, help="tokens per oracle step (reference arm)")
    ap.add_argument("--fp4", action="store_true",
                    help="with a single-layer --workload: its NVFP4 forward on the block-scaled FP4 tensor core")
    ap.add_argument("--tokens", type=int, default=None,
                    help="token batch of the gated-MLP block (default 8192; smaller batches are for profiler captures)")
    args = ap.parse_args()
    CHAIN_TOKENS[0] = args.tokens
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
    if args.workload == CHAIN_WORKLOAD:
        out, ctx = run_ours_chain(args, rank, world, local, peaks)
        out["e2e"] = run_e2e_chain(ctx, args, world)
        dev = ctx[3]
    else:
        out, ctx = run_ours_linear(args, rank, world, local, peaks)
        out["e2e"] = run_e2e_fp4(ctx, args, world) if args.fp4 else run_e2e_linear(ctx, args, world, "grads")
        if ctx[4].backward:
            full = run_e2e_linear(ctx, args, world, "all")
            out["e2e"]["all_outputs"] = {k: full[k] for k in ("value", "ms_per_step", "d2h_bytes_per_step",
                                                              "read_back")}
        dev = ctx[5]
    del ctx
    if rank == 0 and world == 1:
        import torch
        torch.cuda.empty_cache()
        if not args.only_main:
            out["workloads"] = run_other_workloads(peaks, dev)
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
