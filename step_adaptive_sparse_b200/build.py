"""Build libarea.so in-tree with nvcc for sm_100a.

Usage: python -m step_adaptive_sparse_b200.build   (or build() from Python)
The shared library lands in step_adaptive_sparse_b200/lib/libarea.so.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libarea.so")
SOURCES = ["api.cu", "pool_dwt.cu", "plan.cu", "attn_simt.cu", "attn_tc.cu", "noalloc.cu",
           "bridge.cu", "schedule.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


# The window instantiations of attn_tc_kernel (template argument WINDOW =
# true) split their registers with setmaxnreg: 128 threads at 136 and 256 at
# 184, exactly the allocation of 384 threads at 168.  That holds only if
# ptxas gives them 168 registers at entry; the host refuses the launch
# otherwise.  The build checks it here, and that no attention kernel spills.
WINDOW_KERNEL_REGS = 168


def check_attn_resources(ptxas_log: str) -> list[str]:
    """Problems found in ptxas -v output for the attention kernels (empty if none)."""
    problems, name, seen = [], None, 0
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            name = line.split("'")[1] if "'" in line else line
            if "attn_tc_kernel" not in name:
                name = None
            else:
                seen += 1
            continue
        if name is None:
            continue
        if "spill stores" in line:
            parts = line.replace(",", " ").split()
            stores = int(parts[parts.index("spill") - 2])
            loads = int(parts[parts.index("loads") - 3])
            if stores or loads:
                problems.append(f"{name}: {stores} bytes spill stores, {loads} bytes spill loads")
        elif "Used" in line and "registers" in line:
            regs = int(line.split("Used")[1].split()[0])
            window = "attn_tc_kernelILb1E" in name
            if window and regs != WINDOW_KERNEL_REGS:
                problems.append(f"{name}: {regs} registers at entry, the register split needs "
                                f"{WINDOW_KERNEL_REGS}")
            name = None
    if seen == 0:
        problems.append("no attn_tc_kernel instantiation in the ptxas output")
    return problems


def build(verbose: bool = False, jobs: int = 0) -> str:
    """Compile every .cu of csrc/ into lib/libarea.so and return its path."""
    os.makedirs(LIBDIR, exist_ok=True)
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    common = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-ffp-contract=off", "-I", os.path.join(ROOT, "include"),
              "-I", CSRC]
    if verbose:
        common += ["-Xptxas", "-v"]
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = common + ["-c", os.path.join(CSRC, src), "-o", obj]
        if src == "attn_tc.cu" and not verbose:
            cmd[1:1] = ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed.append((src, text))
            continue
        if verbose and text:
            print(f"--- {src}\n{text}", file=sys.stderr)
        if src == "attn_tc.cu":
            problems = check_attn_resources(text)
            if problems:
                failed.append((src, "\n".join(problems)))
    if failed:
        msg = "\n".join(f"--- {s}\n{t}" for s, t in failed)
        raise RuntimeError(f"nvcc failed:\n{msg}")
    link = [nvcc(), *ARCH, "-shared", "-o", LIB, *objs]
    subprocess.run(link, check=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
