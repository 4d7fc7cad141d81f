"""Builds ``libmimo_attn.so`` in-tree with nvcc for sm_100a."""

from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "mimo_attn.cu")
LIB = os.path.join(PKG, "libmimo_attn.so")
# the same sources with every kernel's row indices bounds-checked (-DMIMO_CHECKED)
LIB_CHECKED = os.path.join(PKG, "libmimo_attn_checked.so")
DEPS = [
    os.path.join(PKG, "csrc", f)
    for f in ("mimo_attn.cu", "common.cuh", "decode_kernel.cuh", "prefill_kernel.cuh",
              "prefill_swa_kernel.cuh", "decode_fp8_kernel.cuh",
              "rope_append_kernel.cuh", "decode_merge_kernel.cuh",
              "backward_kernel.cuh", "backward_tc_kernel.cuh", "backward_dq_tc_kernel.cuh")
] + [os.path.join(ROOT, "include", "mimo_attn.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def up_to_date(lib=LIB):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force=False, verbose=False, checked=False):
    """Compile the library (or, with checked=True, its bounds-checked variant) if
    any source is newer than it; returns the .so path."""
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(lib):
        return lib
    extra = ["-DMIMO_CHECKED"] if checked else []
    cmd = [nvcc_path(), *NVCC_FLAGS, *extra, "-Xptxas", "-v", "-o", lib, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stderr)
    return lib


if __name__ == "__main__":
    import sys

    build(force=True, verbose=True, checked="--checked" in sys.argv)
