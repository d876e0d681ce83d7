"""Host-side checks of the benchmark's bookkeeping (no GPU): the kernel-source hash that keys recorded profiler
counters ignores comments but not code, and recorded DRAM traffic is reported only for the code it was taken on."""

import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    b = load_bench()
    csrc = tmp_path / "qlora_fine_tuning_blockwise_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("int f(int a) {\n  return a + 1;  // one\n}\n/* block */\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "LAYER_SOURCES", ("k.cuh",))
    h0 = b.kernel_source_sha()
    (csrc / "k.cuh").write_text("// a new header comment\nint f(int a) {\n    return a + 1;   // changed comment\n}\n")
    assert b.kernel_source_sha() == h0
    (csrc / "k.cuh").write_text("int f(int a) {\n  return a + 2;\n}\n")
    assert b.kernel_source_sha() != h0


def test_recorded_traffic_only_for_matching_code(tmp_path, monkeypatch):
    b = load_bench()
    csrc = tmp_path / "qlora_fine_tuning_blockwise_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("int main() { return 0; }\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "LAYER_SOURCES", ("k.cu",))
    rec = {"source_sha": b.kernel_source_sha(), "workloads": {"wl": {"fused_dx": 123}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert b.load_traffic("wl") == {"fused_dx": 123}
    assert b.load_traffic("other") == {}
    (csrc / "k.cu").write_text("int main() { return 1; }\n")
    assert b.load_traffic("wl") == {}


def test_hashed_sources_are_the_layer_translation_unit():
    """The hash covers exactly qlora.cu and the files it includes (transitively), and no other source: the
    format conversions' kernels (a translation unit of their own) do not make the layer kernels' counters stale."""
    import re
    b = load_bench()
    csrc = os.path.join(ROOT, "qlora_fine_tuning_blockwise_b200", "csrc")
    seen, todo = set(), ["qlora.cu"]
    while todo:
        name = todo.pop()
        if name in seen:
            continue
        seen.add(name)
        text = open(os.path.join(csrc, name)).read()
        todo += [m for m in re.findall(r'#include\s+"([^"/]+)"', text) if os.path.exists(os.path.join(csrc, m))]
    assert seen == set(b.LAYER_SOURCES)
    assert "formats.cu" not in seen


def test_committed_traffic_record():
    """profiles/traffic.json names, per workload, fused kernels with positive byte counts; when it was taken on
    the kernel code in this tree the bench reports it (after a kernel change it is stale and the bench reports
    null)."""
    b = load_bench()
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert rec["workloads"] and all(v > 0 for k in rec["workloads"].values() for v in k.values())
    if rec["source_sha"] != b.kernel_source_sha():
        pytest.skip("traffic recorded before the latest kernel change: re-capture it on a B200")
    for wl, kernels in rec["workloads"].items():
        assert b.load_traffic(wl) == kernels


def test_chain_work_counts():
    """The block's FLOP count is the sum of its three layers' counts, and the four fused GEMMs of a step carry
    the base products (2 M N K each) plus their LoRA products."""
    b = load_bench()
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    M, D, F, r = 8192, 8192, 28672, 64
    gu = I.LinearWorkload("gu", M, D, F, r, 2.0, 0.0)
    dn = I.LinearWorkload("dn", M, F, D, r, 2.0, 0.0)
    ff, fb = b.chain_flops(M, D, F, r)
    assert ff == 2 * gu.flops_fwd + dn.flops_fwd and fb == 2 * gu.flops_bwd + dn.flops_bwd
    k = b.chain_kernel_flops(M, D, F, r)
    assert k["gate_up_fwd"] + k["down_fwd"] == ff - 2 * (2 * M * D * r) - 2 * M * F * r  # minus the s x A^T GEMMs
    assert k["down_dx"] == 2 * M * D * F + 2 * M * r * F and k["gate_up_dx"] == 2 * M * 2 * F * D + 4 * M * r * D
    assert abs(ff / 1e12 - 11.66) < 0.01 and abs(fb / 1e12 - 11.78) < 0.01  # the block's 11.66 / 11.78 TFLOP


def test_clock_summary_parses_samples_and_reasons():
    """nvidia-smi csv lines (noheader, nounits) -> median SM clock, max clock and the active throttle reasons."""
    b = load_bench()
    c = b.ClockSampler(0)
    c.lines = [
        "0, 1800, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1500, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1700.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    c.lines = ["0, 1200, 1965, 500, 0x8, Not Active, Active, Not Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_thermal_slowdown"]
    c.lines = []
    assert c.summary()["reasons"] == ["unsampled"]


def test_flush_l2_writes_then_reads():
    """The flush zeroes its buffer (the write that evicts the workload) and then reads it back."""
    import torch
    b = load_bench()
    buf = torch.full((4096,), 7, dtype=torch.uint8)
    b.flush_l2(buf)
    assert int(buf.sum()) == 0
