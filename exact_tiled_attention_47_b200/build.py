"""Build libfa_sm100.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m exact_tiled_attention_47_b200.build [-v]``.  Each ``csrc/*.cu`` is compiled to an
object under ``_build/`` (skipped when up to date) and the objects are linked into
``exact_tiled_attention_47_b200/lib/libfa_sm100.so`` with the CUDA runtime linked statically, so the
library needs no CUDA shared library at load time (the driver is reached through the runtime).
Kernels that re-split registers between warpgroups (setmaxnreg) are checked against the ptxas report:
the build fails unless they got exactly the register count their source plans for.
"""
from __future__ import annotations

import argparse
import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libfa_sm100.so")
DEBUG_LIB = os.path.join(LIBDIR, "libfa_sm100_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


# Kernels whose warpgroups re-split their registers with setmaxnreg: the split only works when the
# kernel is launched with exactly the register count the source plans for (kLaunchRegs), so the
# build fails if ptxas allocated anything else or spilled.
REGISTER_PLANNED = {"fa_prefill_sm100.cu": ("fa_fwd_kernel", "kLaunchRegs")}


def ptxas_kernels(report: str):
    """{mangled entry name: (registers, spill bytes)} from a ``-Xptxas -v`` report."""
    out, cur = {}, None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            out[cur] = [None, 0]
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            out[cur][1] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            out[cur][0] = int(m.group(1))
    return {k: tuple(v) for k, v in out.items()}


def check_planned_registers(src_name: str, source: str, report: str) -> None:
    """Raise RuntimeError unless every planned kernel of the file got exactly its planned registers."""
    if src_name not in REGISTER_PLANNED:
        return
    kernel, const = REGISTER_PLANNED[src_name]
    m = re.search(r"constexpr int " + const + r" = (\d+);", source)
    if not m:
        raise RuntimeError(f"{src_name}: no '{const}' constant found")
    planned = int(m.group(1))
    found = {k: v for k, v in ptxas_kernels(report).items() if kernel in k}
    if not found:
        raise RuntimeError(f"{src_name}: ptxas reported no {kernel} instantiation")
    bad = {k: v for k, v in found.items() if v[0] != planned or v[1] != 0}
    if bad:
        raise RuntimeError(f"{src_name}: {kernel} must use exactly {planned} registers without spills "
                           f"(setmaxnreg split); ptxas gave {sorted(set(bad.values()))}")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False, debug: bool = False) -> str:
    """Compile and link; returns the library path.  Raises RuntimeError on a compiler error.

    ``debug`` builds ``libfa_sm100_debug.so`` instead: the same sources with ``-DFA_DEBUG`` (index
    checks on every plain global access, reported as FA_ERR_BOUNDS; the prefill walks every key
    block of a causal row instead of skipping the fully masked ones), objects under ``_build/debug``.
    """
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib_path = DEBUG_LIB if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    cc = nvcc()
    headers = _headers()
    srcs = _sources()
    objs = []
    jobs = []
    for src in srcs:
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            planned = os.path.basename(src) in REGISTER_PLANNED
            cmd = ([cc] + ARCH + CFLAGS + (["-DFA_DEBUG"] if debug else []) +
                   (["-Xptxas", "-v"] if (ptxas_info or planned) else []) + ["-c", src, "-o", obj])
            jobs.append((src, obj, cmd))

    def run(job):
        src, obj, cmd = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, cmd, r

    with ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1)) or 1) as ex:
        for src, obj, cmd, r in ex.map(run, jobs):
            if verbose or ptxas_info:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
            try:
                with open(src) as fh:
                    check_planned_registers(os.path.basename(src), fh.read(), r.stdout + r.stderr)
            except RuntimeError:
                os.remove(obj)  # never link (or count as up to date) an object that failed the check
                raise
    if force or jobs or _stale(lib_path, objs):
        cmd = [cc] + ARCH + ["-shared", "-cudart", "static", "-o", lib_path] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if verbose:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return lib_path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills per kernel")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build the index-checking debug library instead")
    a = ap.parse_args()
    print(build(a.verbose, a.ptxas_info, a.force, a.debug))
