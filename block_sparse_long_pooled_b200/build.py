"""Build the CUDA library libfp2.so in-tree for sm_100a (nvcc only; no GPU needed).

Two flavours of the same sources: libfp2.so, and libfp2_checked.so compiled with FP2_CHECKED=1
(device-side hand-off and bounds checks that record FP2_DEV_CHECK; see include/fp2.h)."""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp2.so")
CHECKED_LIB = os.path.join(HERE, "libfp2_checked.so")
SOURCES = ["fp2_api.cu", "pool.cu", "discover.cu", "attention.cu", "fp2_noalloc.cu"]
HEADERS = ["fp2_device.cuh", "fp2_kernels.h", "fp2_plan.h", os.path.join("..", "..", "include", "fp2.h")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def _start(checked: bool, ptxas_info: bool):
    """Launch the nvcc compiles of one flavour; returns (objects, [(cmd, process)])."""
    tmpdir = os.path.join(HERE, "_build_checked" if checked else "_build")
    os.makedirs(tmpdir, exist_ok=True)
    common = [nvcc_path(), "-std=c++17", "-O3", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
              "-I", os.path.join(HERE, "..", "include")]
    if checked:
        common += ["-DFP2_CHECKED=1"]
    if ptxas_info:
        common += ["-Xptxas", "-v"]
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(tmpdir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = common + ["-c", os.path.join(CSRC, src), "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    return objs, procs


def _finish(lib: str, objs, procs, verbose: bool, ptxas_info: bool) -> str:
    for cmd, p in procs:
        out, _ = p.communicate()
        if verbose or ptxas_info or p.returncode != 0:
            sys.stdout.write(out)
        if p.returncode != 0:
            raise RuntimeError("nvcc failed: " + " ".join(cmd))
    tmp_lib = lib + ".tmp"
    link = [nvcc_path(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp_lib] + objs
    subprocess.check_call(link)
    os.replace(tmp_lib, lib)
    return lib


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, checked: bool = False) -> str:
    """Build one flavour (libfp2.so, or libfp2_checked.so with checked=True) if its sources changed."""
    lib = CHECKED_LIB if checked else LIB
    if not force and not needs_build(lib):
        return lib
    objs, procs = _start(checked, ptxas_info)
    return _finish(lib, objs, procs, verbose, ptxas_info)


def build_all(force: bool = False, verbose: bool = False) -> None:
    """Both flavours, compiled side by side."""
    jobs = [(lib, checked) for lib, checked in ((LIB, False), (CHECKED_LIB, True)) if force or needs_build(lib)]
    started = [(lib, *_start(checked, False)) for lib, checked in jobs]
    for lib, objs, procs in started:
        _finish(lib, objs, procs, verbose, False)


if __name__ == "__main__":
    if "--all" in sys.argv:
        build_all(force="--force" in sys.argv, verbose=True)
        print(LIB)
        print(CHECKED_LIB)
    else:
        print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv,
                    checked="--checked" in sys.argv))
