"""Scalar brute-force attention for tiny shapes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Pure-Python loops over (sequence, query, head, key, feature) with ``math.exp``;
no NumPy arithmetic, no blocking.  Same definition as ``oracle.attention``
(MiMo-V2-Flash model doc, "Key features: hybrid attention"; config
``head_dim`` / ``v_head_dim`` / ``num_key_value_heads`` / ``sliding_window``),
written a second time so that one pins the other.  Only for T <= ~32.
"""

from __future__ import annotations

import math


def _tolist(x):
    if hasattr(x, "detach"):
        import torch

        return x.detach().to(dtype=torch.float64).tolist()
    return x.tolist() if hasattr(x, "tolist") else list(x)


def prefill(q, k, v, sinks, window, cu_seqlens, scale):
    """Return (out, lse) as nested lists: out[t][h][e], lse[h][t]."""
    Q, K, V = _tolist(q), _tolist(k), _tolist(v)
    cu = [int(c) for c in _tolist(cu_seqlens)]
    Nt, Hq = len(Q), (len(Q[0]) if Q else 0)
    Hkv = len(K[0]) if K else 1
    G = Hq // Hkv if Hkv else 1
    Dv = len(V[0][0]) if V else 0
    sig = [-math.inf] * Hq if sinks is None else [float(s) for s in _tolist(sinks)]
    out = [[[0.0] * Dv for _ in range(Hq)] for _ in range(Nt)]
    lse = [[-math.inf] * Nt for _ in range(Hq)]
    for s in range(len(cu) - 1):
        b0, b1 = cu[s], cu[s + 1]
        for i in range(b1 - b0):
            for h in range(Hq):
                g = h // G
                scores = []
                for j in range(b1 - b0):
                    d = i - j
                    if d < 0 or (window > 0 and d > window - 1):
                        continue
                    dot = 0.0
                    for c in range(len(Q[b0 + i][h])):
                        dot += Q[b0 + i][h][c] * K[b0 + j][g][c]
                    scores.append((j, scale * dot))
                m = sig[h]
                for _, sc in scores:
                    m = max(m, sc)
                if m == -math.inf:
                    continue
                Z = math.exp(sig[h] - m) if sig[h] != -math.inf else 0.0
                acc = [0.0] * Dv
                for j, sc in scores:
                    w = math.exp(sc - m)
                    Z += w
                    for e in range(Dv):
                        acc[e] += w * V[b0 + j][g][e]
                out[b0 + i][h] = [a / Z for a in acc]
                lse[h][b0 + i] = m + math.log(Z)
    return out, lse
