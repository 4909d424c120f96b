"""Build libzyfa.so (all CUDA kernels + the C ABI) in-tree for sm_100a with nvcc.

    python -m bf16_causal_prefill_fp8_b200.build [--force]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libzyfa.so")
# the same sources with device-side range checks compiled in (a debugging aid:
# every guarded access checks its index first; see zyfa_device_check)
LIB_CHECKED = os.path.join(HERE, "libzyfa_checked.so")
SOURCES = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))]
HEADERS = [os.path.join(ROOT, "include", "zyfa.h")]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]


def _stale(lib) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS + [__file__])


def _compile(lib, extra, verbose):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc] + NVCC_FLAGS + extra + (["-Xptxas", "-v"] if verbose else []) + \
        ["-o", lib + ".tmp", os.path.join(CSRC, "zyfa.cu")]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)


def build(force: bool = False, verbose: bool = False, checked: bool = True) -> str:
    """Builds libzyfa.so and (checked=True) libzyfa_checked.so; returns the
    path of the normal library."""
    if force or _stale(LIB):
        _compile(LIB, [], verbose)
    if checked and (force or _stale(LIB_CHECKED)):
        _compile(LIB_CHECKED, ["-DZYFA_CHECKS"], verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
