"""Build the sm_100a shared library libmmdit.so in-tree with nvcc.

    python -m joint_video_audio_rope_b200.build [--force] [--verbose] [--device-checks]

--device-checks builds the debug variant libmmdit_checked.so instead: kernels
check the indices they read from caller data (block ids and counts, block
tables) on the device and record MMDIT_EDEVCHECK in the device error word
when one is out of range (read back by mmdit_device_status); nothing traps.
Load it by pointing the binding at it (MMDIT_LIB=.../libmmdit_checked.so).

Compiles every .cu file under csrc/ for sm_100a (-gencode
arch=compute_100a,code=sm_100a) with -lineinfo and links them, with the CUDA
runtime linked statically, into joint_video_audio_rope_b200/libmmdit.so.  The
library exports only the C ABI of include/mmdit.h.  nvcc cross-compiles, so
this runs on machines without a GPU.
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
OUT = os.path.join(PKG, "libmmdit.so")
OUT_CHECKED = os.path.join(PKG, "libmmdit_checked.so")
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps.append(os.path.join(ROOT, "include", "mmdit.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          device_checks: bool = False) -> str:
    out = OUT_CHECKED if device_checks else OUT
    if not force and not _stale(out):
        return out
    bdir = os.path.join(BUILD, "checked") if device_checks else BUILD
    os.makedirs(bdir, exist_ok=True)
    defs = ["-DMMDIT_DEVICE_CHECKS"] if device_checks else []
    objs, cmds = [], []
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *ARCH, *FLAGS, *defs, "-c", src, "-o", obj]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        cmds.append(cmd)
        objs.append(obj)
    # the translation units are independent: compile them concurrently
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
        for r in ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds):
            if r.stdout or r.stderr:
                print(r.stdout + r.stderr, end="", flush=True)
            r.check_returncode()
    tmp = out + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-Xcompiler", "-fPIC"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--device-checks", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_verbose=a.ptxas_verbose,
                device_checks=a.device_checks))
    sys.exit(0)
