"""Builds libvdn.so in-tree with nvcc for sm_100a (B200).

Usage: python -m linear_attention_video_block_b200.build [--verbose-ptxas] [--checked]

--checked builds libvdn_checked.so instead: the same sources with
-DVDN_BOUND_CHECKS, whose kernels check their global row / slot / chunk
indices and the schedule's key rows before each access and, on a failed check,
skip the access and record VDN_ERR_BOUNDS in the device status word (no trap).
It is a debugging aid; the regular library has no checks.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libvdn.so")
LIB_CHECKED = os.path.join(PKG, "libvdn_checked.so")
SOURCES = ["vdn_abi.cu", "window_simt.cu", "window_tc.cu", "window_fp8.cu", "gram_tc.cu", "vda.cu",
           "readout.cu", "readout_tc.cu", "combine.cu", "vda_noalloc.cu", "host_pipeline.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xcompiler", "-Wall", "-diag-suppress", "177"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, verbose_ptxas: bool, checked: bool = False) -> str:
    sub = os.path.join(BUILD, "checked") if checked else BUILD
    obj = os.path.join(sub, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-DVDN_BOUND_CHECKS"] if checked else []), "-c",
           os.path.join(CSRC, src), "-o", obj]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose_ptxas: bool = False, checked: bool = False) -> str:
    os.makedirs(os.path.join(BUILD, "checked") if checked else BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, checked), SOURCES))
    out = LIB_CHECKED if checked else LIB
    tmp = out + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, checked="--checked" in sys.argv))
