"""Build libtri.so (the sm_100a CUDA library behind include/tri.h) in-tree.

    python -m rope_aware_kv_b200.build [--verbose]

Compiles every ``csrc/*.cu`` with nvcc for ``sm_100a`` (-gencode
arch=compute_100a,code=sm_100a, -lineinfo) and links them into
``rope_aware_kv_b200/libtri.so`` with the CUDA runtime linked statically, so
the library depends on nothing but the driver.  Rebuilds only when a source
or header is newer than the library.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtri.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; set NVCC or install the CUDA toolkit")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, jobs: int = 8, out: str = LIB,
          defines=()) -> str:
    """Compile the library to ``out`` (default: the in-tree libtri.so); extra
    ``-D`` defines select compile-time variants of the kernels."""
    if out == LIB and not defines and not force and not _stale():
        return LIB
    nvcc = _nvcc()
    tmp = tempfile.mkdtemp(prefix="tri_build_")
    try:
        objs = []
        procs = []
        for src in sources():
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [nvcc, *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-c", src,
                   "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                                stderr=subprocess.STDOUT, text=True)))
            objs.append(obj)
            if len(procs) >= jobs:
                _drain(procs, verbose)
        _drain(procs, verbose)
        tmp_out = out + ".tmp"
        subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp_out, *objs], check=True)
        os.replace(tmp_out, out)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    return out


def _drain(procs, verbose):
    failed = []
    while procs:
        src, p = procs.pop(0)
        out, _ = p.communicate()
        if verbose or p.returncode:
            sys.stdout.write(f"--- {os.path.basename(src)}\n{out}")
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(os.path.basename(f) for f in failed))


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
