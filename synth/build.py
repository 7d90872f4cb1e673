"""Compile the seeded input generator: host (gcc) and device (nvcc, sm_100a)."""
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(verbose: bool = False, device: bool = True) -> None:
    host = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-o",
            os.path.join(HERE, "libsynth_host.so"), os.path.join(HERE, "synth_host.c")]
    if verbose:
        print(" ".join(host))
    subprocess.run(host, check=True)
    if not device:
        return
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    dev = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-o", os.path.join(HERE, "libsynth_dev.so"),
           os.path.join(HERE, "synth_dev.cu")]
    if verbose:
        print(" ".join(dev))
    subprocess.run(dev, check=True)


if __name__ == "__main__":
    build(verbose=True)
