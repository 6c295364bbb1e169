"""Build libgkd.so (the CUDA kernels + C ABI) in-tree for sm_100a.

    python -m prompt_conditioned_keypoint_b200.build [--verbose-ptxas]

Compiles every csrc/*.cu with nvcc into prompt_conditioned_keypoint_b200/libgkd.so
(cudart linked statically, so the library needs only the NVIDIA driver at run
time). Rebuilds only when a source or header is newer than the library.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgkd.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False, trace_to: str | None = None) -> str:
    """Build libgkd.so. `trace_to` builds a separate timeline-tracing variant
    (-DGKD_TRACE, exports gkd_trace_read) at that path instead."""
    out = trace_to or LIB
    if trace_to is None and not force and not verbose_ptxas and not _stale():
        return LIB
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-o", out + ".tmp", *sources()]
    if trace_to is not None:
        cmd.insert(1, "-DGKD_TRACE")
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
    if verbose_ptxas:
        sys.stderr.write(proc.stdout + proc.stderr)
    os.replace(out + ".tmp", out)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--trace-to", default=None, help="build the tracing variant at this path")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas, trace_to=args.trace_to))


if __name__ == "__main__":
    main()
