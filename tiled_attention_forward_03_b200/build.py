"""Build the in-tree shared library ``libattn_fwd.so`` (CUDA, sm_100a only).

``python -m tiled_attention_forward_03_b200.build`` compiles
``csrc/attn_api.cu`` (which includes the kernel) with nvcc into the package
directory, next to this file, so the library travels with the source tree.
The build checks ptxas's register report: the kernel's warpgroup register
split assumes a fixed register count at launch, and any other count is
rejected here as well as at run time.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libattn_fwd.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
SOURCES = ["attn_api.cu"]
HEADERS = ["attn_fwd_kernel.cuh", "attn_fwd_colsplit_kernel.cuh", "attn_fwd_wide_kernel.cuh", "attn_bwd_kernel.cuh", "attn_rope_kernel.cuh", "sm100_ptx.cuh"]
EXPECTED_REGS = 168

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-shared", "-Xcompiler", "-fPIC,-O2",
    "-Xptxas", "-v",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the attention library")


def have_nvcc() -> bool:
    try:
        _nvcc()
        return True
    except RuntimeError:
        return False


def _inputs() -> list[str]:
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "attn.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if any input is newer than it; return its path."""
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC,
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    log = proc.stdout + proc.stderr
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + log)
    # register count of each forward-kernel instance (bf16 D = 32/64/96/128, bf16 D = 32/64 with
    # P beside O, E4M3 D = 32/64/96/128), of the column-split kernel (D = 32/64/96/128) and of the
    # backward kernels at D = 32/64/128 (both passes): all use the same warpgroup register split
    # (the self-test kernels and the 320-thread backward at D = 96 are exempt)
    regs, spills, current = [], [], None
    split_kernel = lambda name: ("attn_fwd_sm100" in name or "attn_fwd_colsplit_sm100" in name
                                 or ("attn_bwd_sm100" in name and "ILi96E" not in name))
    for line in log.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            current = m.group(1)
        m = re.search(r"Used (\d+) registers", line)
        if m and current and split_kernel(current):
            regs.append(int(m.group(1)))
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and current and split_kernel(current):
            spills.append(int(m.group(1)))
    if len(regs) != 20 or any(r != EXPECTED_REGS for r in regs):
        os.remove(tmp)
        raise RuntimeError(f"unexpected kernel register counts {regs} (want {EXPECTED_REGS}):\n{log}")
    if verbose:
        print(log)
        print(f"registers {regs}, spill stores {spills}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH



# The files that define each measured path's kernels and their launch: a traffic record taken
# with ncu stays valid while these files are unchanged.
DIGEST_FILES = {
    "fwd": ["attn_fwd_colsplit_kernel.cuh", "attn_fwd_kernel.cuh", "sm100_ptx.cuh", "attn_api.cu"],
    "wide": ["attn_fwd_wide_kernel.cuh", "attn_fwd_kernel.cuh", "sm100_ptx.cuh", "attn_api.cu"],
    "bwd": ["attn_bwd_kernel.cuh", "attn_fwd_kernel.cuh", "sm100_ptx.cuh", "attn_api.cu"],
    "all": SOURCES + HEADERS,
}


def kernel_source_digest(which: str = "all") -> str:
    """SHA-256 over the CUDA sources of one path ("fwd", "bwd") or of all ("all"); identifies
    the kernels an ncu capture measured."""
    import hashlib
    h = hashlib.sha256()
    for name in DIGEST_FILES[which]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, verbose=True)
    print(path)
