"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (bf16 inputs, fp32 accumulation): max-abs error <= 1e-2 and
relative Frobenius error <= 5e-3 against the fp64 oracle; LSE within 1e-3.
Where a bf16 output can exceed |4| (tiny windows, where the output is one
value row times a probability), the bf16 rounding of the output itself is
up to 2^-9 |ref|, so the max-abs bound there is 1e-2 + 2^-8 |ref|.
"""

import numpy as np
import torch

MAX_ABS = 1e-2
REL_FRO = 5e-3
LSE_ABS = 1e-3


def to64(t):
    return t.detach().to(device="cpu", dtype=torch.float64).numpy()


def check(out_gpu, out_ref, lse_gpu=None, lse_ref=None, rel_term=True, what=""):
    o = to64(out_gpu)
    assert o.shape == out_ref.shape, (o.shape, out_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - out_ref)
    bound = MAX_ABS + (2.0 ** -8) * np.abs(out_ref) if rel_term else MAX_ABS
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"{what}: max-abs {err.max():.3e} at {worst}"
    den = np.linalg.norm(out_ref)
    if den > 0:
        rel = np.linalg.norm(o - out_ref) / den
        assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e}"
    if lse_gpu is not None:
        l = to64(lse_gpu)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness differs"
        d = np.abs(l[fin] - lse_ref[fin])
        assert d.size == 0 or d.max() <= LSE_ABS, f"{what}: lse err {d.max():.3e}"


def strict(out_gpu, out_ref, lse_gpu=None, lse_ref=None, what=""):
    """The benchmark spec's tolerance exactly: max-abs 1e-2, rel-Frobenius 5e-3."""
    check(out_gpu, out_ref, lse_gpu, lse_ref, rel_term=False, what=what)
