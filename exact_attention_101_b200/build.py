"""Build the CUDA library ``libfa_b200.so`` in-tree for sm_100a.

``python -m exact_attention_101_b200.build`` (or ``build()``) compiles
``csrc/fa_api.cu`` with nvcc into ``exact_attention_101_b200/libfa_b200.so``; the
Python binding in ``__init__.py`` loads that file.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfa_b200.so")
SOURCES = [os.path.join(CSRC, "fa_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("fa_fwd_kernel.cuh", "fa_fwd_pair.cuh", "fa_bwd_kernel.cuh",
                                                  "fa_quant.cuh", "sm100.cuh")] + [
    os.path.join(ROOT, "include", "fa_b200.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than any of its sources."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(f) <= t for f in DEPS):
            return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    extra = os.environ.get("FA_NVCC_EXTRA", "").split()  # e.g. tuning -D overrides
    cmd = [_nvcc()] + NVCC_FLAGS + extra + ["-I", os.path.join(ROOT, "include"), "-I", CSRC,
                                             "-o", tmp] + SOURCES
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libfa_b200.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
