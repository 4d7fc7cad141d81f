"""FP8 (e4m3) KV-cache decode for the fp64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

MiMo-V2-Flash model doc, "Key features": the model is trained with FP8 mixed
precision.  The pages do not define a KV-cache format, so this library's own
reading is used: every cache element is an e4m3 code times one fp32 scale per
key/value head (one scale for K, one for V, per layer).

e4m3 (the OCP 8-bit floating-point format E4M3): bit 7 is the sign, bits 6..3
the exponent ``e`` with bias 7, bits 2..0 the mantissa ``m``; there are no
infinities, and ``e = 15, m = 7`` is NaN:

    e = 0:       value = (-1)^s * (m / 8) * 2^-6          (subnormal)
    e = 1..15:   value = (-1)^s * (1 + m / 8) * 2^(e - 7)  (largest finite 448)

The decode itself is ``attention.decode`` on the dequantised caches.
"""

from __future__ import annotations

import numpy as np

from .attention import decode


def e4m3_to_float(codes):
    """float64 values of e4m3 codes (uint8 array or tensor), from the format definition."""
    if hasattr(codes, "detach"):
        import torch

        codes = codes.detach().to("cpu").view(torch.uint8).numpy()
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * mag
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)


def decode_fp8(q, k_codes, v_codes, k_scale, v_scale_kv, seqlens, window, sinks, ring=None,
               scale=None, v_scale=1.0, batch_index=None):
    """One decode step per sequence over e4m3 caches with per-KV-head scales (float64).

    Same arguments and results as ``attention.decode``, except that the caches
    hold e4m3 codes ``[B, C, Hkv, D]`` and ``k_scale`` / ``v_scale_kv`` ``[Hkv]``
    give each head's scale: a key element is ``code * k_scale[g]``.
    """
    C = k_codes.shape[1]
    if ring is None:
        ring = window > 0 and C == window
    ks = np.asarray(_np(k_scale), dtype=np.float64).reshape(1, -1, 1)
    vs = np.asarray(_np(v_scale_kv), dtype=np.float64).reshape(1, -1, 1)
    Ls = np.asarray(_np(seqlens), dtype=np.int64).reshape(-1)
    idx = range(len(Ls)) if batch_index is None else [int(b) for b in np.asarray(batch_index).reshape(-1)]
    outs, lses = [], []
    for b in idx:
        L = int(Ls[b])
        n = max(0, min(L, C))  # slots that hold tokens (ring: the most recent min(L, C))
        kd = e4m3_to_float(k_codes[b, :n]) * ks
        vd = e4m3_to_float(v_codes[b, :n]) * vs
        # one sequence, truncated to its valid slots; the ring/linear reading
        # is the full cache's (a truncated ring of L <= C slots is position order)
        o, l = decode(q[b:b + 1], kd[None], vd[None], np.array([L]), window, sinks, ring=ring,
                      scale=scale, v_scale=v_scale)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def _np(x):
    if hasattr(x, "detach"):
        return x.detach().to("cpu").numpy()
    return np.asarray(x)
