"""Compile the C oracle (fp64 and fp32 copies) into shared libraries beside
this file.  Test infrastructure only."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "vsa_oracle.c")
VARIANTS = {
    "f64": [],
    "f32": ["-DREAL=float", "-DORACLE_EXP=expf", "-DORACLE_SQRT=sqrtf"],
}


def lib_path(precision: str) -> str:
    return os.path.join(HERE, f"liboracle_{precision}.so")


def build(force: bool = False) -> None:
    for prec, defs in VARIANTS.items():
        out = lib_path(prec)
        if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
            continue
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *defs,
               "-o", tmp, SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, out)


if __name__ == "__main__":
    build(force="--force" in sys.argv)
