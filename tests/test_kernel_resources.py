"""Build health of the CUDA sources for sm_100a, checked on the CPU: every
kernel and device function compiles without register spills, and the fused
decode kernel (512 threads, one block per SM) stays within 128 registers per
thread with no stack frame, as does the grouped tensor-core kernel (480
threads: four warps share a sub-partition's 16,384 registers, so a launch with
more than 128 a thread fails).  A spill in these kernels costs far more than any
tuning gains, so it should fail here rather than show up as a slowdown.
(Only ptxas's resource summary is read.)"""
import concurrent.futures
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantised_expert_ffn_router_b200", "csrc")


def _ptxas_report(nvcc, src, out_dir):
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                        "--expt-relaxed-constexpr", "-Xptxas", "-v", "-c", src, "-o", obj],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stderr


def _functions(report):
    """(function name, registers, stack bytes, spill store bytes, spill load bytes) per compiled function."""
    out, name, stack, spills = [], None, 0, (0, 0)
    for line in report.splitlines():
        m = re.search(r"(?:Compiling entry function|Function properties for) '?([\w$]+)'?", line)
        if m:
            name = m.group(1)
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            stack, spills = int(m.group(1)), (int(m.group(2)), int(m.group(3)))
            out.append((name, None, stack, *spills))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            out.append((name, int(m.group(1)), stack, *spills))
    return out


def test_no_spills_and_decode_register_budget(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    sources = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(sources)) as pool:
        reports = dict(zip(sources, pool.map(lambda s: _ptxas_report(nvcc, s, str(tmp_path)), sources)))
    decode_entries = 0
    for src, rep in reports.items():
        for name, regs, stack, st, ld in _functions(rep):
            assert st == 0 and ld == 0, f"{os.path.basename(src)}: {name} spills ({st} B stored, {ld} B loaded)"
            if "bt_tc_gemm_kernel" in name and regs is not None:
                # 15 warps: an SM sub-partition holds four of them in its 16,384 registers
                assert regs <= 128, f"{name}: {regs} registers (4 warps x 32 x 128 per sub-partition)"
            if "decode_kernel" in name and regs is not None:
                decode_entries += 1
                assert regs <= 128, f"{name}: {regs} registers (512 threads x 128 fill the SM)"
                assert stack == 0, f"{name}: {stack} B stack frame"
    assert decode_entries == 4  # <4|2 bits> x <single-layer | multi-layer>
