"""Builds libhardkv.so (sm_100a) in-tree with nvcc, and its bounds-checked twin
libhardkv_checked.so (-DHARDKV_CHECKED: every checked index that is out of range sets
HARDKV_DEV_CHECK in the status words and the access is skipped; no traps)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libhardkv.so")
LIB_CHECKED = os.path.join(HERE, "libhardkv_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]
VARIANTS = {LIB: [], LIB_CHECKED: ["-DHARDKV_CHECKED"]}


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def up_to_date(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(HERE, "..", "include", "hardkv.h")]
    return all(os.path.getmtime(s) <= t for s in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/hardkv_api.cu (which includes every kernel) into libhardkv.so and
    libhardkv_checked.so (two nvcc processes at once); returns the first's path."""
    jobs = {}
    for lib, extra in VARIANTS.items():
        if force or not up_to_date(lib):
            cmd = [NVCC, *FLAGS, *extra, "-o", lib + ".tmp", os.path.join(CSRC, "hardkv_api.cu")]
            jobs[lib] = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                         text=True)
    for lib, proc in jobs.items():
        out, err = proc.communicate()
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + out + err)
        os.replace(lib + ".tmp", lib)
        if verbose and lib == LIB:
            sys.stderr.write(err)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
