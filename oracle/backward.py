"""Gradients of the sliding-window / global attention with a sink, fp64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The forward is ``attention.prefill`` (MiMo-V2-Flash model doc, "Key
features": hybrid attention with a *learnable* attention-sink bias, so the
sink logit has a gradient).  Per query head h, query row i and its visible
keys j, with S_ij = s <q_i, k_j>, lse_i including the sink and
P_ij = exp(S_ij - lse_i):

    O_i      = v_scale * sum_j P_ij v_j
    dP_ij    = v_scale * <dO_i, v_j>
    D_i      = <dO_i, O_i>                       (= sum_j P_ij dP_ij)
    dS_ij    = P_ij (dP_ij - D_i)
    dq_i     = s * sum_j dS_ij k_j
    dk_j    += s * sum_i dS_ij q_i               (over the query heads of k's group)
    dv_j    += v_scale * sum_i P_ij dO_i         (same)
    dsigma_h = - sum_i exp(sigma_h - lse_i) D_i

(the sink is a softmax entry with no value: its own dP is 0, so its
gradient is its probability times (0 - D_i)).  Everything is computed from
the definition with explicit probability matrices, one (sequence, head) at a
time; the tests pin it to central finite differences of the forward.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import _f64, _i64, visible


def prefill_backward(q, k, v, do, sinks, window, cu_seqlens, scale=None, v_scale=1.0):
    """Returns (dq [Nt,Hq,Dqk], dk [Nt,Hkv,Dqk], dv [Nt,Hkv,Dv], dsinks [Hq] or None), float64."""
    qd, kd, vd, dod = _f64(q), _f64(k), _f64(v), _f64(do)
    Nt, Hq, Dqk = qd.shape
    Hkv = kd.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    sig = np.full(Hq, -np.inf) if sinks is None else _f64(sinks).reshape(Hq)
    cu = _i64(cu_seqlens).reshape(-1)
    dq = np.zeros_like(qd)
    dk = np.zeros_like(kd)
    dv = np.zeros_like(vd)
    ds = np.zeros(Hq)
    for b0, b1 in zip(cu[:-1], cu[1:]):
        n = int(b1 - b0)
        if n == 0:
            continue
        pos = np.arange(n)
        mask = visible(pos[:, None], pos[None, :], window)         # [i, j]
        for h in range(Hq):
            g = h // G
            Q = qd[b0:b1, h]
            K = kd[b0:b1, g]
            V = vd[b0:b1, g]
            dO = dod[b0:b1, h]
            S = np.where(mask, scale * (Q @ K.T), -np.inf)
            m = np.maximum(S.max(axis=1), sig[h])
            e = np.where(mask, np.exp(S - m[:, None]), 0.0)
            sink = np.exp(sig[h] - m) if np.isfinite(sig[h]) else np.zeros(n)
            Z = e.sum(axis=1) + sink
            P = e / Z[:, None]                                       # rows sum with the sink to 1
            O = v_scale * (P @ V)
            dP = v_scale * (dO @ V.T)
            D = (dO * O).sum(axis=1)
            dS = P * (dP - D[:, None])
            dq[b0:b1, h] += scale * (dS @ K)
            dk[b0:b1, g] += scale * (dS.T @ Q)
            dv[b0:b1, g] += v_scale * (P.T @ dO)
            ds[h] -= float(((sink / Z) * D).sum())
    return dq, dk, dv, (None if sinks is None else ds)


def _row_block(qd, kd, vd, dod, sig, h, g, r0, r1, window, scale, v_scale):
    """Rows r0..r1-1 of one sequence and query head h: the keys they can see
    start at k_lo; returns k_lo, P [rows, keys k_lo..r1-1], dP, D, lse."""
    k_lo = 0 if window == 0 else max(0, r0 - window + 1)
    rows = np.arange(r0, r1)
    keys = np.arange(k_lo, r1)
    mask = visible(rows[:, None], keys[None, :], window)
    Q = qd[r0:r1, h]
    K = kd[k_lo:r1, g]
    V = vd[k_lo:r1, g]
    dO = dod[r0:r1, h]
    S = np.where(mask, scale * (Q @ K.T), -np.inf)
    m = np.maximum(S.max(axis=1), sig[h])
    e = np.where(mask, np.exp(S - m[:, None]), 0.0)
    sink = np.exp(sig[h] - m) if np.isfinite(sig[h]) else np.zeros(len(rows))
    Z = e.sum(axis=1) + sink
    P = e / Z[:, None]
    O = v_scale * (P @ V)
    dP = v_scale * (dO @ V.T)
    D = (dO * O).sum(axis=1)
    return k_lo, P, dP, D, m + np.log(Z)


def prefill_backward_sampled(q, k, v, do, sinks, window, q_rows, q_heads, k_rows, kv_heads,
                             sink_heads=(), scale=None, v_scale=1.0, block=512):
    """Gradients of ONE sequence ([n, H, D] tensors) at sampled positions, each
    from its own rows of P (same definitions as ``prefill_backward``), for
    sizes where the full gradients are out of reach:

      dq [len(q_rows), len(q_heads), Dqk]   at query rows x query heads
      dk [len(k_rows), len(kv_heads), Dqk]  at key rows x KV heads (summed over the group)
      dv [len(k_rows), len(kv_heads), Dv]
      ds [len(sink_heads)]                  dsigma_h (every row of head h)

    A key's gradient needs every query row that sees it, so key rows are
    cheap only under a window or near the end of the sequence.
    """
    qd, kd, vd, dod = _f64(q), _f64(k), _f64(v), _f64(do)
    n, Hq, Dqk = qd.shape
    Hkv = kd.shape[1]
    G = Hq // Hkv
    Dv = vd.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    sig = np.full(Hq, -np.inf) if sinks is None else _f64(sinks).reshape(Hq)
    dq = np.zeros((len(q_rows), len(q_heads), Dqk))
    for a, i in enumerate(q_rows):
        for b, h in enumerate(q_heads):
            k_lo, P, dP, D, _ = _row_block(qd, kd, vd, dod, sig, h, h // G, i, i + 1, window, scale,
                                           v_scale)
            dS = P[0] * (dP[0] - D[0])
            dq[a, b] = scale * (dS @ kd[k_lo:i + 1, h // G])
    dk = np.zeros((len(k_rows), len(kv_heads), Dqk))
    dv = np.zeros((len(k_rows), len(kv_heads), Dv))
    for a, j in enumerate(k_rows):
        i_hi = n if window == 0 else min(n, j + window)  # query rows that see key j: [j, i_hi)
        for b, g in enumerate(kv_heads):
            for h in range(g * G, (g + 1) * G):
                for r0 in range(j, i_hi, block):
                    r1 = min(i_hi, r0 + block)
                    k_lo, P, dP, D, _ = _row_block(qd, kd, vd, dod, sig, h, g, r0, r1, window, scale,
                                                   v_scale)
                    pj = P[:, j - k_lo]
                    dS = pj * (dP[:, j - k_lo] - D)
                    dk[a, b] += scale * (dS @ qd[r0:r1, h])
                    dv[a, b] += v_scale * (pj @ dod[r0:r1, h])
    ds = np.zeros(len(sink_heads))
    for b, h in enumerate(sink_heads):
        if not np.isfinite(sig[h]):
            continue
        for r0 in range(0, n, block):
            r1 = min(n, r0 + block)
            _, _, _, D, lse = _row_block(qd, kd, vd, dod, sig, h, h // G, r0, r1, window, scale, v_scale)
            ds[b] -= float((np.exp(sig[h] - lse) * D).sum())
    return dq, dk, dv, ds
