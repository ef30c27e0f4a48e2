"""Build libllvq.so (the CUDA library behind include/llvq.h) in-tree with nvcc for sm_100a."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libllvq.so")
SOURCES = [os.path.join(CSRC, f) for f in ("llvq.cu", "tables.cpp", "tables96.cpp")]
HEADERS = [os.path.join(CSRC, f) for f in ("tables.h", "tables96.h", "device_common.cuh", "codec48.cuh", "codec72.cuh",
                                            "codec96.cuh", "encode48.cuh", "encode72.cuh", "encode96.cuh", "kernels.cuh", "kernels_bin48.cuh", "kernels_tc.cuh",
                                            "kernels_tc48.cuh", "kernels_gemv48.cuh", "search48.cuh", "search48_classes.cuh", "gptq48.cuh")] + [os.path.join(ROOT, "include", "llvq.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-pthread", "-shared", "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"), "-o", tmp, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libllvq.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
