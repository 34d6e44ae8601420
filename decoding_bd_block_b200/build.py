"""Build libbd.so in-tree with nvcc for sm_100a (B200).

    python -m decoding_bd_block_b200.build [--force]

Compiles every ``csrc/*.cu`` into ``decoding_bd_block_b200/libbd.so``
(static CUDA runtime, no torch dependency), and the same sources with the
device-side index checks (``-DBD_DEVICE_CHECKS``) into ``libbd_checks.so``.
Rebuilds only when a source or header is newer than the library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbd.so")
# the same sources with the device-side index checks compiled in (diagnostics)
LIB_CHECKS = os.path.join(PKG, "libbd_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + [os.path.join(ROOT, "include", "bd.h"), os.path.abspath(__file__)])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _command(lib: str, extra, verbose: bool):
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr", *extra,
           "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp", *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    return cmd


def build(force: bool = False, verbose: bool = False, checks: bool = True) -> str:
    """Build libbd.so and (checks=True) libbd_checks.so, the two compilations
    running side by side; returns libbd.so's path."""
    jobs = [(LIB, [])] + ([(LIB_CHECKS, ["-DBD_DEVICE_CHECKS"])] if checks else [])
    procs = [(lib, subprocess.Popen(_command(lib, extra, verbose)))
             for lib, extra in jobs if force or not up_to_date(lib)]
    failed = [lib for lib, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(failed)})")
    for lib, _ in procs:
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
