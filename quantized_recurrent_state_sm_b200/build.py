"""Build the CUDA library libstepq.so (sm_100a) in-tree with nvcc."""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libstepq.so")
# the checking build (kernels validate the pool's tables before touching
# memory; see stepq_pool_check_guards in include/stepq.h)
LIB_CHECK = os.path.join(HERE, "libstepq_check.so")
SOURCES = ["stepq_abi.cu", "stepq_kernels.cu"]
HEADERS = ["stepq_internal.cuh", "stepq_device.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    out = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    out.append(os.path.join(ROOT, "include", "stepq.h"))
    return out


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    """Build libstepq.so, or with check=True the checking build libstepq_check.so
    (-DSTEPQ_CHECK=1)."""
    lib = LIB_CHECK if check else LIB
    if not (force or needs_build(lib)):
        return lib
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", lib + ".tmp"]
    if check:
        cmd.append("-DSTEPQ_CHECK=1")
    if verbose:
        cmd.append("-Xptxas=-v")
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, check="--check" in sys.argv))
