"""Builds ``libmoe_b200.so`` in-tree with nvcc for sm_100a.

    python -m mixture_experts_routed_03_b200.build [--force]

The library is one translation unit (``csrc/moe_api.cu`` includes the kernel
headers); the runtime is linked statically and the driver's tensor-map
encoder is looked up at run time, so the .so needs no libcuda at link time.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libmoe_b200.so")
SOURCES = ["moe_api.cu"]
# the tensor-core peak probe the benchmark reports its roofline against
PEAK_OUT = os.path.join(HERE, "libmoe_peak.so")
PEAK_SOURCES = ["mma_peak.cu"]
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _deps():
    """Every CUDA source and header of the library, and the C header."""
    return sorted(os.path.join(CSRC, n) for n in os.listdir(CSRC)
                  if n.endswith((".cu", ".cuh", ".h"))) + [HEADER]


def up_to_date(out=OUT):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    deps = _deps()
    return all(os.path.getmtime(d) <= t for d in deps)


def _compile(out, sources, log_name):
    cmd = [_nvcc()] + NVCC_FLAGS + ["-o", out] + [os.path.join(CSRC, s) for s in sources]
    res = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    log = res.stdout + res.stderr
    with open(os.path.join(HERE, log_name), "w") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log[-4000:])
    return log


def build(force=False, verbose=False):
    """Compile the libraries that are missing or older than their sources;
    returns the path of the layer's library."""
    for out, sources, log_name in ((OUT, SOURCES, "build.log"), (PEAK_OUT, PEAK_SOURCES, "build_peak.log")):
        if force or not up_to_date(out):
            log = _compile(out, sources, log_name)
            if verbose:
                print(log)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
