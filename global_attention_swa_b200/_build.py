"""Builds ``libmimo_attn.so`` in-tree with nvcc for sm_100a."""

from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "mimo_attn.cu")
LIB = os.path.join(PKG, "libmimo_attn.so")
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


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force=False, verbose=False):
    """Compile the library if any source is newer than it; returns the .so path."""
    if not force and up_to_date():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-Xptxas", "-v", "-o", LIB, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose=True)
