"""Build libmla.so in-tree with nvcc for sm_100a.

    python -m mla_latent_kv_42_b200.build [--verbose] [--force]

The library is one translation unit (csrc/libmla.cu) compiled with
``-gencode arch=compute_100a,code=sm_100a``; it links only the CUDA runtime (static). The same
source is also built with MLA_FAULT_INJECT into libmla_faultinj.so, the test build whose waits
give up after 20 ms and which can leave a cache load unissued (mla_debug_inject_missing_load);
only the bounded-wait test loads it.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmla.so")
LIB_FAULTINJ = os.path.join(PKG, "libmla_faultinj.so")


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h")))


def up_to_date(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")] + [__file__]
    return all(os.path.getmtime(p) <= t for p in deps)


def _nvcc_cmd(lib: str, defines: list[str], verbose: bool) -> list[str]:
    cmd = [
        nvcc(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-shared",
        "-I", INCLUDE, "-I", CSRC, *defines,
        os.path.join(CSRC, "libmla.cu"),
        "-o", lib + ".tmp",
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False, faultinj: bool = True) -> str:
    """Build libmla.so (and, unless faultinj is False, the fault-injection test build, in
    parallel); return the path of libmla.so."""
    jobs = [(LIB, [], verbose)]
    if faultinj:
        jobs.append((LIB_FAULTINJ, ["-DMLA_FAULT_INJECT"], False))
    running = []
    for lib, defines, verb in jobs:
        if force or not up_to_date(lib):
            cmd = _nvcc_cmd(lib, defines, verb)
            running.append((lib, cmd, verb, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                                             text=True)))
    for lib, cmd, verb, proc in running:
        out, err = proc.communicate()
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + out + err)
        if verb:
            sys.stderr.write(out + err)
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose))
