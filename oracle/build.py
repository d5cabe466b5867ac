"""Build the CPU oracle (test infrastructure only).

Compiles hgd_oracle.c three times with gcc: libhgd_oracle.so (double
arithmetic), libhgd_oracle_f32.so (float arithmetic) and libhgd_oracle_omp.so
(double, its GEMV and dense state product spread over the host's cores with
OpenMP; the all-cores CPU baseline).  -O2 -ffp-contract=off and no
fast-math keep every sum in the order the source writes it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hgd_oracle.c")
TARGETS = {
    "libhgd_oracle.so": [],
    "libhgd_oracle_f32.so": ["-DHGDO_FP32", "-DHGDO_REAL=float"],
    # the same loops with their output elements shared out over the host's cores
    # (each element's sum in the same order: the same results as the first build)
    "libhgd_oracle_omp.so": ["-fopenmp"],
}


def build(force: bool = False) -> None:
    for name, defs in TARGETS.items():
        out = os.path.join(HERE, name)
        deps = [SRC, os.path.join(HERE, "hgd_oracle.h"), __file__]
        if not force and os.path.exists(out) and all(
                os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
            continue
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-fno-semantic-interposition",
               "-shared", "-Wall", "-Wextra", "-Wno-unused-parameter", "-Wno-unknown-pragmas", *defs, SRC,
               "-o", out + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)


if __name__ == "__main__":
    build(force=True)
