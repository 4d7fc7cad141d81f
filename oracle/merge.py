"""Merging decode results computed over disjoint parts of a cache, fp64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

A global layer's decode attends to every cached key, and softmax with a sink
is a sum over keys, so the keys may be split into disjoint parts (one per
GPU, "context parallelism"): part r yields its plain-softmax result without
the sink, ``out_r`` and ``lse_r = ln sum_{j in r} exp(S_j)``.  With
``M = max(sigma, max_r lse_r)``:

    Z   = exp(sigma - M) + sum_r exp(lse_r - M)
    out = v_scale * sum_r exp(lse_r - M) out_r / Z
    lse = M + ln Z

which equals the decode over all keys with the sink (MiMo-V2-Flash model doc,
"Key features": learnable attention sink; the sink reading of
``oracle/attention.py``).  A part with no keys has ``lse_r = -inf``; it is
left out of both sums, whatever its ``out_r`` holds.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import _f64


def merge(part_out, part_lse, sinks, v_scale=1.0):
    """part_out [R, B, Hq, Dv], part_lse [R, B, Hq] -> (out [B, Hq, Dv], lse [B, Hq]), float64."""
    po = _f64(part_out)
    pl = _f64(part_lse)
    R, B, Hq = pl.shape
    sig = np.full(Hq, -np.inf) if sinks is None else _f64(sinks).reshape(Hq)
    out = np.zeros(po.shape[1:])
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            M = max(sig[h], pl[:, b, h].max())
            if not np.isfinite(M):
                continue
            live = np.isfinite(pl[:, b, h])   # a part without keys contributes nothing
            w = np.exp(pl[live, b, h] - M)
            Z = w.sum() + (math.exp(sig[h] - M) if np.isfinite(sig[h]) else 0.0)
            out[b, h] = v_scale * (w @ po[live, b, h, :]) / Z
            lse[b, h] = M + math.log(Z)
    return out, lse
