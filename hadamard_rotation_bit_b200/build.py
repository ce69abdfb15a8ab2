"""Build libhadq.so in-tree with nvcc for sm_100a.

    python -m hadamard_rotation_bit_b200.build [--force] [--verbose]

The shared library lands next to this file, where the ctypes binding looks
for it.  Only nvcc is needed (cross-compiles without a GPU).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libhadq.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ARCH_FLAGS + [
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]
LINK_FLAGS = ARCH_FLAGS + ["--shared", "-cudart", "static", "-Xcompiler", "-fvisibility=hidden"]

# Translation units: the host side (validation, launch planning, C ABI) and
# one unit per kernel family, compiled in parallel.
UNITS = ["hadq_api.cu", "kernels_segment.cu", "kernels_team.cu", "kernels_team_bf16.cu", "kernels_tc.cu",
         "kernels_tck.cu", "kernels_ksize.cu", "kernels_ksize_bf16.cu", "hadq_codebook.cu"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh", ".h"))] + [
        os.path.join(INCLUDE, "hadq.h")]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}): {' '.join(cmd[-3:])}\n{res.stderr[-8000:]}")
    return res.stderr


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile libhadq.so if it is missing or older than its sources; return its path."""
    if not force and not needs_build():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    nvcc = _nvcc()
    with tempfile.TemporaryDirectory(prefix="hadq_build_") as tmp:
        objs, cmds = [], []
        for unit in UNITS:
            obj = os.path.join(tmp, unit.replace(".cu", ".o"))
            cmd = [nvcc] + COMPILE_FLAGS + ["-I", INCLUDE, "-I", CSRC]
            if ptxas_info:
                cmd += ["-Xptxas", "-v"]
            cmds.append(cmd + ["-c", os.path.join(CSRC, unit), "-o", obj])
            objs.append(obj)
        with ThreadPoolExecutor(max_workers=len(cmds)) as ex:
            logs = list(ex.map(lambda c: _run(c, verbose), cmds))
        if verbose or ptxas_info:
            for log in logs:
                print(log, file=sys.stderr)
        _run([nvcc] + LINK_FLAGS + objs + ["-o", LIB + ".tmp"], verbose)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills per kernel")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    main()
