"""Build libcsa2.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

The CUDA runtime is linked statically and the driver's tensor-map encoder is fetched at run
time, so the library loads on a machine without a GPU driver (only device calls need one).
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
OUT = os.path.join(HERE, "libcsa2.so")
BUILD = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date():
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force=False, verbose=False, jobs=8):
    if not force and up_to_date():
        return OUT
    os.makedirs(BUILD, exist_ok=True)
    objs, procs = [], []
    for src in _sources():
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = [NVCC] + ARCH + FLAGS + (["-Xptxas", "-v"] if verbose else []) + \
            ["-dc" if False else "-c", src, "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
        if len(procs) >= jobs:
            _drain(procs, verbose)
    _drain(procs, verbose)
    link = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", OUT + ".tmp"] + objs + \
        ["-Xlinker", "--exclude-libs,ALL"]
    subprocess.check_call(link)
    os.replace(OUT + ".tmp", OUT)
    return OUT


def _drain(procs, verbose):
    while procs:
        cmd, p = procs.pop(0)
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            sys.stderr.write(text)
            raise RuntimeError("nvcc failed: " + " ".join(cmd))
        if verbose and text.strip():
            sys.stderr.write(text)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
