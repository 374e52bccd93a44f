"""Build the sm_100a shared library libmuon_b200.so in the package directory.

nvcc compiles every .cu under csrc/ for sm_100a (B200) only; cudart is linked
statically, the driver API is reached through cudaGetDriverEntryPoint, so
the library loads on a machine without a GPU (its calls then return errors).
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmuon_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "-I", os.path.join(ROOT, "include"), "-I", CSRC,
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in deps())


def build(force=False, verbose=False, extra=()):
    if not force and up_to_date():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    builddir = os.path.join(HERE, "_build")
    os.makedirs(builddir, exist_ok=True)
    jobs = []
    for src in sources():
        obj = os.path.join(builddir, os.path.basename(src) + ".o")
        cmd = [NVCC, "-c", src, "-o", obj] + [f for f in FLAGS if f != "-shared"] + list(extra)
        if verbose:
            print(" ".join(cmd))
        jobs.append((cmd, obj))
    # one nvcc per translation unit, in parallel
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as pool:
        for f in [pool.submit(subprocess.check_call, cmd) for cmd, _ in jobs]:
            f.result()
    objs = [obj for _, obj in jobs]
    cmd = [NVCC, "-shared", "-o", LIB + ".tmp"] + objs + ["-gencode", "arch=compute_100a,code=sm_100a",
                                                           "-cudart", "static", "-Xcompiler", "-fPIC"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
