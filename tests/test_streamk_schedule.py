"""The fused GEMM's stream-K schedule (token-light forward) is a partition of the work (CPU only).

tests/streamk_schedule.cu compiles the kernel's own schedule functions for the host and walks them over the
decode layer's shape and a few hundred random (tiles, stages per tile, CTAs): every stage of every tile is done
once, a tile's parts come from consecutive CTAs in order with slabs 0, 1, ... -- as many as the reduction sums --,
the LoRA stages run once per tile, and the CTAs' stage counts differ by at most one.  A planted mistake (one CTA
walking the schedule of a grid one CTA larger) must make every case fail.
"""

import os
import shutil
import subprocess

import pytest


def test_streamk_schedule_is_a_balanced_partition(tmp_path):
    nvcc = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = os.path.join(str(tmp_path), "streamk_schedule")
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "streamk_schedule.cu")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "--expt-relaxed-constexpr",
                    "-o", exe, src], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    lines = r.stdout.strip().splitlines()
    assert r.returncode == 0, [l for l in lines if l.startswith("FAIL")][:5]
    assert len(lines) == 308 and all(l.startswith("ok ") for l in lines)
    # the checker catches a schedule walked with the wrong grid size on one CTA
    r = subprocess.run([exe, "planted"], capture_output=True, text=True)
    lines = r.stdout.strip().splitlines()
    assert r.returncode == 0 and not any(l.startswith("ok ") for l in lines), [l for l in lines if l.startswith("ok")][:3]
