"""Builds the CUDA libraries in-tree (sm_100a): block_denoising_step_b200/lib/libdgen.so, the
denoising path, and lib/libdgen_probe.so, the same sources plus the GEMM-core measurement
probes of include/dgen_probe.h (used only by bench.py's --gemm-* measurements)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIB_DIR, "libdgen.so")
PROBE_LIB = os.path.join(LIB_DIR, "libdgen_probe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-O3",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(os.path.join(SRC_DIR, f) for f in os.listdir(SRC_DIR) if f.endswith((".cu", ".cuh")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    hdrs = [os.path.join(ROOT, "include", h) for h in ("dgen.h", "dgen_probe.h")]
    return any(os.path.getmtime(s) > t for s in sources() + hdrs)


def _compile(lib: str, defines, verbose: bool, extra) -> None:
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *defines, *extra, "-I", os.path.join(ROOT, "include"), "-I", SRC_DIR, "-o", tmp,
           os.path.join(SRC_DIR, "dgen.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=(), probes: bool = True) -> str:
    """Compiles libdgen.so (and, with probes, libdgen_probe.so) when a source changed."""
    if force or needs_build(LIB):
        _compile(LIB, [], verbose, extra)
    if probes and (force or needs_build(PROBE_LIB)):
        _compile(PROBE_LIB, ["-DDGEN_PROBES"], verbose, extra)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else (), probes="--no-probes" not in sys.argv)
