"""Build libvdit_attn.so in-tree with nvcc for sm_100a.

``python -m video_diffusion_transformer_attention_b200.build`` (or
``__graft_entry__.build()``) compiles ``csrc/vdit_attn.cu`` into
``libvdit_attn.so`` next to this file.  No GPU is needed to build.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libvdit_attn.so")
SOURCES = [os.path.join(CSRC, f) for f in ("vdit_attn.cu", "attn_fwd_sm100.cuh", "sm100_ptx.cuh",
                                           "attn_merge.cuh", "qk_norm.cuh", "fp8_quant.cuh",
                                           "attn_fwd_fp8_sm100.cuh", "sm100_fp8_ptx.cuh", "vsmooth_group.cuh",
                                           "attn_cross_sm100.cuh", "attn_cross_fp8_sm100.cuh")]
HEADERS = [os.path.join(INCLUDE, "vdit_attn.h"), os.path.join(INCLUDE, "vdit_attn_testing.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def _launch_regs_expected() -> int:
    src = open(os.path.join(CSRC, "attn_fwd_sm100.cuh")).read()
    return int(re.search(r"kLaunchRegs\s*=\s*(\d+)", src).group(1))


def check_launch_registers(ptxas_log: str) -> int:
    """The forward kernel re-splits its registers with setmaxnreg, which is only
    safe if ptxas allocated exactly kLaunchRegs a thread at launch; a smaller
    allocation would leave setmaxnreg.inc waiting forever.  Returns the count."""
    found = re.findall(r"Compiling entry function '(\w*attn_fwd_\w*kernel\w*)'.*?Used (\d+) registers",
                       ptxas_log, flags=re.S)
    if not found:
        raise RuntimeError("could not find the forward kernel's register count in the ptxas output")
    expected = _launch_regs_expected()
    for name, used in found:
        if int(used) != expected:
            raise RuntimeError(f"{name} allocates {used} registers a thread, "
                               f"the setmaxnreg split assumes {expected}")
    return expected


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-Xptxas=-v", *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "vdit_attn.cu"), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libvdit_attn.so")
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    try:
        check_launch_registers(res.stderr)
    except RuntimeError:
        os.unlink(tmp)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
