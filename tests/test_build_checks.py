"""The build's register check for kernels that re-split registers with setmaxnreg (CPU only).

The prefill kernel is launched with kLaunchRegs registers per thread and then moves them between
warpgroups; if ptxas allocated a different count the split would not add up and the kernel could not
run.  build.py therefore parses the ptxas report of that file and fails the build unless every
instantiation got exactly the planned count without spills.  These tests feed the check reports with
the right count, another count and a spill, and run it on the real compiler output.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from exact_tiled_attention_47_b200 import build  # noqa: E402

SRC = "constexpr int kLaunchRegs = 168;\n"


def report(regs, spill=0, name="_ZN2fa13fa_fwd_kernelILi64ELb0ELb0EEEv"):
    return (f"ptxas info    : Compiling entry function '{name}' for 'sm_100a'\n"
            f"ptxas info    : Function properties for {name}\n"
            f"    0 bytes stack frame, {spill} bytes spill stores, {spill} bytes spill loads\n"
            f"ptxas info    : Used {regs} registers, used 1 barriers\n")


def test_parser_reads_registers_and_spills():
    k = build.ptxas_kernels(report(168) + report(96, 8, name="other_kernel"))
    assert k == {"_ZN2fa13fa_fwd_kernelILi64ELb0ELb0EEEv": (168, 0), "other_kernel": (96, 16)}


def test_planned_count_passes():
    build.check_planned_registers("fa_prefill_sm100.cu", SRC, report(168) + report(168, name="x_fa_fwd_kernel_y"))


@pytest.mark.parametrize("rep", [report(160), report(168, spill=4), report(168) + report(176, name="fa_fwd_kernel2"), ""])
def test_other_counts_spills_or_nothing_fail(rep):
    with pytest.raises(RuntimeError):
        build.check_planned_registers("fa_prefill_sm100.cu", SRC, rep)


def test_unplanned_files_are_not_checked():
    build.check_planned_registers("fa_decode_sm100.cu", "", report(40))


def test_real_prefill_object_passes_the_check():
    src = os.path.join(build.CSRC, "fa_prefill_sm100.cu")
    r = subprocess.run([build.nvcc()] + build.ARCH + build.CFLAGS + ["-Xptxas", "-v", "-c", src, "-o", os.devnull],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    with open(src) as fh:
        build.check_planned_registers("fa_prefill_sm100.cu", fh.read(), r.stdout + r.stderr)
