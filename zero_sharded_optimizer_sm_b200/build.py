"""Build step of the ZeRO step library: ``libzero_sm.so`` for sm_100a.

nvcc cross-compiles without a GPU.  Floating-point flags keep every device
operation IEEE-conformant (no fast-math, no flush to zero, correctly rounded
division and square root, no multiply-add contraction) so that the kernels'
arithmetic is the one stated in ``csrc/kernels.cu``.
"""
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = ["csrc/zero_api.cu", "csrc/kernels.cu", "csrc/fused_tma.cu", "csrc/fused_bulk.cu", "csrc/static_scratch.cu",
           "csrc/two_pass_tma.cu", "csrc/dist.cu", "csrc/guards.cu",
           "csrc/plan.cpp"]
LIB = os.path.join(HERE, "libzero_sm.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
    "-Xcompiler", "-fPIC",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    return shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


def build(verbose: bool = False, ptxas_verbose: bool = False) -> str:
    from concurrent.futures import ThreadPoolExecutor

    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    cmds, objs = [], []
    for src in SOURCES:
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *NVCC_FLAGS]
        if src.endswith(".cpp"):
            cmd += ["-x", "cu"]
        cmd += ["-c", os.path.join(HERE, src), "-o", obj]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd))
        cmds.append(cmd)
        objs.append(obj)
    # the translation units are independent: compile them side by side
    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as pool:
        for res in pool.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds):
            if verbose or ptxas_verbose or res.returncode != 0:
                print(res.stdout, end="")
                print(res.stderr, end="")
            if res.returncode != 0:
                raise subprocess.CalledProcessError(res.returncode, res.args, res.stdout, res.stderr)
    # link beside the library and rename over it: a reader never sees a
    # half-written file
    tmp = LIB + ".tmp"
    link = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs]
    if verbose:
        print(" ".join(link))
    subprocess.run(link, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys

    print(build(verbose=True, ptxas_verbose="-v" in sys.argv))
