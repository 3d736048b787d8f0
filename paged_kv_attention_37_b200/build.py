"""Build the CUDA library in place: paged_kv_attention_37_b200/libpkv.so.

One translation unit (csrc/pkv_api.cu includes the kernels), compiled for
sm_100a only, with the CUDA runtime linked statically so the library loads
without a GPU driver present (the driver API is reached at run time through
cudaGetDriverEntryPoint).

    python paged_kv_attention_37_b200/build.py [--verbose]

(Run it by path: importing the package itself loads the library.)
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpkv.so")
SOURCES = [os.path.join(CSRC, "pkv_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(os.path.dirname(HERE), "include", "pkv.h")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or put CUDA's bin directory on PATH")


def command(out: str = LIB, ptxas_verbose: bool = False, defines=()) -> list[str]:
    cmd = [nvcc_path(), *[f"-D{d}" for d in defines], "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-shared", "--cudart", "static", "-o", out]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    return cmd + SOURCES


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = command(tmp, ptxas_verbose=verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
