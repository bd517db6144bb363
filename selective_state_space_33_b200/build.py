"""Build libsscan.so (the CUDA library behind include/sscan.h) in-tree for sm_100a."""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsscan.so")
# the same library with the index checks of csrc/sscan_check.cuh compiled in
LIB_DEBUG = os.path.join(HERE, "libsscan_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                              + glob.glob(os.path.join(ROOT, "include", "*.h")))


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every .cu under csrc/ into one shared library (sm_100a only).

    debug=True builds libsscan_debug.so instead: the same kernels with every computed
    index into a workspace, parameter or state array checked (SSCAN_DEBUG_BOUNDS); a bad
    index raises bit 3 of the device status word and the access is skipped.  It is
    compiled with relocatable device code so that all kernels share that word."""
    out = LIB_DEBUG if debug else LIB
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(p) for p in deps())
        if os.path.getmtime(out) >= newest:
            return out
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", out + ".tmp"] + sources()
    if debug:
        cmd[1:1] = ["-DSSCAN_DEBUG_BOUNDS=1", "-rdc=true"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
