"""Comparison helpers for GPU-vs-oracle parity tests.

Stated tolerance (bf16 inputs, fp32 accumulation): max-abs error <= 1e-2 and
relative Frobenius error <= 5e-3 against the fp64 oracle; LSE within 1e-3.

``check`` applies exactly that bound to fp32 outputs.  A bf16 output is the
kernel's fp32 result rounded to nearest-even once more, on its way out; that
rounding moves a value by at most half a bf16 unit in the last place (ulp) at
its magnitude, which for |out| >= 2.56 alone exceeds 1e-2.  So a bf16 output
element may differ by 1e-2 plus half an ulp at |ref| + 1e-2 (the magnitude of
the kernel's value before rounding, at most); nothing else is added, for P or
anything else.
"""

import numpy as np
import torch

MAX_ABS = 1e-2
REL_FRO = 5e-3
LSE_ABS = 1e-3


def to64(t):
    return t.detach().to(device="cpu", dtype=torch.float64).numpy()


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits): the most that
    round-to-nearest-even moves a value of that magnitude."""
    _, e = np.frexp(np.abs(np.asarray(x, dtype=np.float64)))  # |x| = m 2^e, m in [0.5, 1)
    return np.ldexp(1.0, e - 9)


def output_bound(out_dtype, ref):
    """Per-element bound on |out - ref| for an output of ``out_dtype``."""
    if out_dtype == torch.bfloat16:
        return MAX_ABS + bf16_half_ulp(np.abs(ref) + MAX_ABS)
    return np.full(np.shape(ref), MAX_ABS)


def check(out_gpu, out_ref, lse_gpu=None, lse_ref=None, what=""):
    """The stated bound (plus the bf16 output's own rounding); returns max-abs."""
    o = to64(out_gpu)
    assert o.shape == out_ref.shape, (o.shape, out_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - out_ref)
    bound = output_bound(out_gpu.dtype, out_ref)
    if err.size:
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        assert np.all(err <= bound), (
            f"{what}: max-abs {err.max():.3e}; worst vs bound at {worst}: "
            f"err {err[worst]:.3e} bound {bound[worst]:.3e} ref {out_ref[worst]:.4f}")
    den = np.linalg.norm(out_ref)
    if den > 0:
        relf = np.linalg.norm(o - out_ref) / den
        assert relf <= REL_FRO, f"{what}: rel-Frobenius {relf:.3e}"
    if lse_gpu is not None:
        l = to64(lse_gpu)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness differs"
        d = np.abs(l[fin] - lse_ref[fin])
        assert d.size == 0 or d.max() <= LSE_ABS, f"{what}: lse err {d.max():.3e}"
    return float(err.max()) if err.size else 0.0
