"""Compile the CPU oracle into ``oracle/liboracle.so`` with gcc.

The oracle is test infrastructure: building it is part of ``build()`` so that
the oracle is ready, but only the tests, the smoke check and the benchmark's
CPU-baseline / reference arm load it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sage_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

# -ffp-contract=off and no fast-math: every float expression in the oracle is
# a single IEEE binary32 operation rounded to nearest-even.
CFLAGS = ["-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-pthread", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def build_variant(defines, out_dir=None) -> str:
    """Compile a separate copy of the oracle with extra preprocessor defines
    (``{"ORC_PLANT": 2}``, ``{"ORC_PSCALE_UNFOLDED": 1}``) for the tests that
    show which mistakes or alternative readings the pins detect.  The default
    library is never replaced."""
    import tempfile
    tag = "_".join("%s%s" % (k, v) for k, v in sorted(defines.items()))
    out_dir = out_dir or os.path.join(tempfile.gettempdir(), "sage_oracle_variants")
    os.makedirs(out_dir, exist_ok=True)
    path = os.path.join(out_dir, "liboracle_%s.so" % tag)
    if os.path.exists(path) and os.path.getmtime(path) >= os.path.getmtime(SRC):
        return path
    tmp = path + ".tmp%d" % os.getpid()
    flags = ["-D%s=%s" % (k, v) for k, v in sorted(defines.items())]
    subprocess.run(["gcc", *CFLAGS, *flags, SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
