"""Rotary position embedding and the decode-step cache append, fp64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

MiMo-V2-Flash model doc: ``MiMoV2FlashConfig.rope_parameters`` (a dictionary
holding ``rope_theta``) and ``MiMoV2FlashModel.forward`` (``position_ids``,
``past_key_values``).  The pages fix neither the value of theta nor how the
rotation pairs dimensions; the reading used here is the rotary embedding of
RoFormer in the rotate-half arrangement: for the first ``rotary_dim`` (even)
dimensions, dimension ``i < rotary_dim / 2`` pairs with ``i + rotary_dim / 2``
and both turn by the angle ``p * theta ** (-2 i / rotary_dim)`` at position p:

    x'[i]         = x[i] cos(a) - x[i + d/2] sin(a)
    x'[i + d/2]   = x[i + d/2] cos(a) + x[i] sin(a)

Dimensions at or past ``rotary_dim`` are left as they are.  The operator's
``q``/``k`` are taken after this rotation; the decode step rotates the new
token's query and key and writes its key and value into the cache slot of
position ``p = L - 1`` (``p mod C`` for a ring of ``C`` slots).
"""

from __future__ import annotations


import numpy as np

from .attention import _f64


def rope_angles(positions, theta, rotary_dim):
    """[n, rotary_dim / 2] angles p * theta^(-2i / rotary_dim), float64."""
    if rotary_dim % 2:
        raise ValueError("rotary_dim must be even")
    half = rotary_dim // 2
    i = np.arange(half, dtype=np.float64)
    inv = np.power(float(theta), -2.0 * i / rotary_dim)
    return np.asarray(positions, dtype=np.float64).reshape(-1, 1) * inv.reshape(1, -1)


def rope(x, positions, theta, rotary_dim=None):
    """Rotate the last axis of ``x`` [n, ..., D] at per-row positions [n] (float64)."""
    x = _f64(x)
    D = x.shape[-1]
    d = D if rotary_dim is None else int(rotary_dim)
    if d > D or d < 0:
        raise ValueError("rotary_dim out of range")
    out = x.copy()
    if d == 0:
        return out
    ang = rope_angles(positions, theta, d)                      # [n, d/2]
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (d // 2,)
    c = np.cos(ang).reshape(shape)
    s = np.sin(ang).reshape(shape)
    a = x[..., : d // 2]
    b = x[..., d // 2: d]
    out[..., : d // 2] = a * c - b * s
    out[..., d // 2: d] = b * c + a * s
    return out


def append_slot(L, capacity, ring):
    """Cache slot of the newest token when ``L`` tokens exist (it is at position L - 1)."""
    p = int(L) - 1
    if p < 0:
        raise ValueError("a sequence needs at least its new token")
    if ring:
        return p % capacity
    if p >= capacity:
        raise ValueError("linear cache is full")
    return p


def rope_append(q, k_new, v_new, k_cache, v_cache, seqlens, window, theta, rotary_dim=None):
    """One decode step's rotation and cache write, float64.

    Args:
      q [B, Hq, Dqk], k_new [B, Hkv, Dqk], v_new [B, Hkv, Dv]: the new token's
        projections before rotation.
      k_cache [B, C, Hkv, Dqk], v_cache [B, C, Hkv, Dv]: caches (copied, not modified).
      seqlens [B]: tokens including the new one (its position is L - 1).
      window: ring cache iff window > 0 and C == window.

    Returns (q_rot, k_cache', v_cache') as float64 arrays.
    """
    qd, kd, vd = _f64(q), _f64(k_new), _f64(v_new)
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    C = kc.shape[1]
    ring = window > 0 and C == window
    Ls = np.asarray(_f64(seqlens), dtype=np.int64).reshape(-1)
    pos = Ls - 1
    q_rot = rope(qd, pos, theta, rotary_dim)
    k_rot = rope(kd, pos, theta, rotary_dim)
    for b, L in enumerate(Ls):
        slot = append_slot(L, C, ring)
        kc[b, slot] = k_rot[b]
        vc[b, slot] = vd[b]
    return q_rot, kc, vc


__all__ = ["rope", "rope_angles", "rope_append", "append_slot"]
