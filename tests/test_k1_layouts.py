"""Host-side check of K1's layouts (no GPU): tests/host/k1_layout_check.cu is
compiled with nvcc against the kernel header and run on the CPU.  It uses the
header's own constexpr layout functions to check, for every (K, values per
thread) the kernels instantiate, that each register/thread layout covers the
row one-to-one and that every 16-byte shared-memory exchange access is free of
bank conflicts, with writer and reader addressing each element identically.
tests/host/k1_expand_plan_check.cu checks, the same way, how the large-batch
forward's K1 shares out the widening of the packed weights over its groups
(every chunk exactly once) and which shapes its routing rule gives it."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_k1_layouts_bijective_and_conflict_free():
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "k1_layout_check")
    src = os.path.join(ROOT, "tests", "host", "k1_layout_check.cu")
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    r = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-x", "cu", "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "hadamard_rotated_int4_b200", "csrc"),
                        "-o", exe, src], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    lines = run.stdout.strip().splitlines()
    assert len(lines) == 12, run.stdout
    assert run.returncode == 0 and all(l.endswith(": ok") for l in lines), run.stdout


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_k1_weight_expansion_plan():
    # tests/host/k1_expand_plan_check.cu: the word widening against the
    # packing's definition, every chunk of the packed weights widened exactly
    # once by K1's groups, and the rule that takes the expansion into K1
    # picking the expected shapes
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "k1_expand_plan_check")
    src = os.path.join(ROOT, "tests", "host", "k1_expand_plan_check.cu")
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    r = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-x", "cu", "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "hadamard_rotated_int4_b200", "csrc"),
                        "-o", exe, src], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    lines = run.stdout.strip().splitlines()
    assert len(lines) == 1 + 10 + 7 * 4 * 4, run.stdout
    assert run.returncode == 0 and all(l.endswith(": ok") for l in lines), run.stdout
