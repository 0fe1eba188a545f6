"""Builds the sm_100a CUDA library ``libnsa_sel.so`` in the package directory.

nvcc cross-compiles without a GPU.  The C ABI is declared in ``include/nsa_sel.h``.
Run ``python -m block_sparse_attention_selected_b200.build`` or call ``build()``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnsa_sel.so")
# the bounds-checking build (-DNSA_SEL_CHECKS): same ABI, every gathered row and K/V
# block coordinate checked before its copy (nsa_common.cuh)
LIB_CHECKS = os.path.join(HERE, "libnsa_sel_checks.so")
SOURCES = ["api.cu", "invert.cu", "fwd.cu", "merge.cu", "bwd.cu", "select.cu", "bsfa.cu"]
HEADERS = ["nsa_common.cuh", "nsa_kernels.h"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "nsa_sel.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    """Builds libnsa_sel.so (checks=True: the bounds-checking libnsa_sel_checks.so)."""
    lib = LIB_CHECKS if checks else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(HERE, "_build_checks" if checks else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    procs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [_nvcc(), *NVCC_FLAGS, *(["-DNSA_SEL_CHECKS"] if checks else []), "-I",
               os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        procs.append((subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT), src))
        objs.append(obj)
    failed = []
    for p, src in procs:
        out, _ = p.communicate()
        if p.returncode != 0 or verbose:
            sys.stderr.write(out.decode(errors="replace"))
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-o", tmp, *objs])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                checks="--checks" in sys.argv))
