"""Build libmoeinputs.so: host generator (g++, no FP contraction) + device
generator (nvcc, sm_100a) in one shared library, in-tree."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _run(cmd):
    print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "csrc")
    out = os.path.join(HERE, "libmoeinputs.so")
    deps = [os.path.join(src, f) for f in os.listdir(src)] + [__file__]
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    host_o = os.path.join(bdir, "gen_host.o")
    dev_o = os.path.join(bdir, "gen_device.o")
    _run(["g++", "-std=c++17", "-O2", "-fPIC", "-ffp-contract=off", "-fno-fast-math", "-pthread",
          "-c", os.path.join(src, "gen_host.cpp"), "-o", host_o])
    _run([NVCC, *ARCH, "-O3", "-lineinfo", "-fmad=false", "-std=c++17", "-Xcompiler", "-fPIC",
          "-c", os.path.join(src, "gen_device.cu"), "-o", dev_o])
    _run([NVCC, *ARCH, "-shared", "-o", out, host_o, dev_o, "-Xcompiler", "-pthread"])
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv)
