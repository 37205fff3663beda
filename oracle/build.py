"""Build the fp64 CPU oracle (test infrastructure) as a shared library.

Compiles ``attn_oracle.c`` (attention), ``quant_oracle.c`` (fp8 quantisation with
incoherent processing), ``bwd_oracle.c`` (gradients) and ``dropout_oracle.c`` (dropout and
its Philox generator) with gcc and OpenMP into ``oracle/liboracle.so``.  Only the
tests, the smoke check and the CPU-baseline leg of ``bench.py`` load that library.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_oracle.c")
QUANT_SRC = os.path.join(HERE, "quant_oracle.c")
BWD_SRC = os.path.join(HERE, "bwd_oracle.c")
DROPOUT_SRC = os.path.join(HERE, "dropout_oracle.c")
SOURCES = (SRC, QUANT_SRC, BWD_SRC, DROPOUT_SRC)
LIB = os.path.join(HERE, "liboracle.so")


def compile_library(out: str, sources, opt: str = "-O2") -> None:
    """gcc the given oracle sources into the shared library ``out``."""
    cmd = ["gcc", opt, "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", out] + list(sources) + ["-lm"]
    subprocess.run(cmd, check=True)


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than one of its sources."""
    if (not force and os.path.exists(LIB)
            and all(os.path.getmtime(LIB) >= os.path.getmtime(s) for s in SOURCES)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    compile_library(tmp, SOURCES)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
