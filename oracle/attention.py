"""fp64 CPU oracle: sliding-window / global causal GQA attention with a sink.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What is computed, and where it comes from
-----------------------------------------
MiMo-V2-Flash model doc, "Key features" (hybrid attention bullet): sliding
window attention (SWA) and global attention (GA) layers interleave 5:1, the
window is aggressive (prose: 128 tokens) and a *learnable attention sink bias*
keeps long-context quality.  ``MiMoV2FlashConfig`` parameters: 64 query heads
(``num_attention_heads``) share 4 key/value heads (``num_key_value_heads``,
grouped-query attention); ``head_dim=192`` is the query/key dimension and
``v_head_dim=128`` the value dimension; ``sliding_window=129``.

Readings taken where the documentation is silent (each one is stated once
here and tested in ``tests/test_oracle_pins.py``):

* window ``W`` counts the query itself: key ``j`` is visible to query ``i`` of
  the same sequence iff ``0 <= i - j`` and (``W == 0`` or ``i - j <= W - 1``).
  ``W = 129`` is "the query plus the previous 128 keys", reconciling the prose
  (128-token window) with the config (``sliding_window=129``); ``W = 0`` means
  global (full causal) attention.
* scale ``s = 1/sqrt(head_dim) = 1/sqrt(192)``.
* query head ``h`` reads key/value head ``h // (Hq / Hkv)`` (consecutive groups,
  the usual grouped-query reading of ``num_key_value_heads``).
* sink: one logit ``sigma_h`` per query head, in natural-log units, not
  multiplied by ``s``; it enters only the normaliser:

      m   = max(sigma_h, max_j S_j)
      Z   = exp(sigma_h - m) + sum_j exp(S_j - m)
      out = sum_j exp(S_j - m) v_j / Z
      lse = m + ln Z                       (natural log, includes the sink)

  ``sinks=None`` means no sink (``sigma = -inf``): plain softmax.  A row with
  no visible key and no sink gives ``out = 0``, ``lse = -inf``.
* ``attention_value_scale`` (0.707) is a linear constant; it is exposed as
  ``v_scale`` (default 1.0) and multiplies the output.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

#: ``1/sqrt(head_dim)`` with ``head_dim = 192`` (``MiMoV2FlashConfig``).
DEFAULT_SCALE_DQK = 1.0 / math.sqrt(192.0)

_ROW_BLOCK = 256


def _f64(x):
    """Convert a NumPy array or torch tensor (any float dtype) to float64 NumPy."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: bf16 has no NumPy dtype
        import torch

        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _blas_threads(n):
    try:
        from threadpoolctl import threadpool_limits

        return threadpool_limits(limits=n, user_api="blas")
    except Exception:  # pragma: no cover - threadpoolctl missing
        import contextlib

        return contextlib.nullcontext()


def _i64(x):
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


def visible(i, j, window):
    """Visibility of key position ``j`` to query position ``i`` (same sequence).

    Causal plus, for ``window > 0``, at most ``window - 1`` keys back.
    Works elementwise on NumPy arrays.
    """
    d = np.asarray(i) - np.asarray(j)
    ok = d >= 0
    if window > 0:
        ok = ok & (d <= window - 1)
    return ok


def _softmax_with_sink(S, sigma):
    """Rows of scores ``S`` ([n, m], -inf where not visible) and one sink logit.

    Returns the weights ``exp(S - m) / Z`` (sink mass excluded) and ``lse``.
    """
    n = S.shape[0]
    rowmax = S.max(axis=1) if S.shape[1] > 0 else np.full(n, -np.inf)
    m = np.maximum(rowmax, sigma)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_safe[:, None])  # exp(-inf) = 0 for masked entries
    Z = E.sum(axis=1) + np.exp(sigma - m_safe)
    with np.errstate(divide="ignore", invalid="ignore"):
        W = np.where(Z[:, None] > 0, E / np.where(Z > 0, Z, 1.0)[:, None], 0.0)
        lse = np.where(Z > 0, m_safe + np.log(np.where(Z > 0, Z, 1.0)), -np.inf)
    return W, lse


def _row_blocks(qpos_sorted):
    """Runs of sorted query positions spanning fewer than _ROW_BLOCK positions."""
    n = len(qpos_sorted)
    start = 0
    for i in range(1, n + 1):
        if (i == n or qpos_sorted[i] - qpos_sorted[start] >= _ROW_BLOCK
                or i - start >= _ROW_BLOCK):
            yield start, i
            start = i


def _one_head(q_h, K, V, qpos, kpos, window, sigma, scale):
    """All requested query rows of one head against one sequence's keys."""
    n = q_h.shape[0]
    out = np.zeros((n, V.shape[1]))
    lse = np.full(n, -np.inf)
    order = np.argsort(qpos, kind="stable")
    qs = qpos[order]
    for r0, r1 in _row_blocks(qs):
        idx = order[r0:r1]
        ip = qs[r0:r1]
        # keys that can be visible to any row of the block
        lo = 0 if window == 0 else max(0, int(ip.min()) - window + 1)
        hi = int(ip.max()) + 1
        kp = kpos[lo:hi]
        S = scale * (q_h[idx] @ K[lo:hi].T)
        S = np.where(visible(ip[:, None], kp[None, :], window), S, -np.inf)
        Wt, l = _softmax_with_sink(S, sigma)
        out[idx] = Wt @ V[lo:hi]
        lse[idx] = l
    return out, lse


def prefill(q, k, v, sinks, window, cu_seqlens, scale=None, v_scale=1.0,
            rows=None, threads=None):
    """Packed (varlen) prefill attention, float64.

    Args:
      q: [Nt, Hq, Dqk]; k: [Nt, Hkv, Dqk]; v: [Nt, Hkv, Dv] (any float type;
         bf16 torch tensors are read exactly).
      sinks: [Hq] sink logits, or None for no sink.
      window: 0 = global causal; >= 1 = query plus previous ``window - 1`` keys.
      cu_seqlens: [num_seqs + 1] cumulative lengths, cu[0] = 0.
      scale: softmax scale, default ``1/sqrt(Dqk)``.
      v_scale: constant multiplier on the output (``attention_value_scale``).
      rows: optional packed token indices; only those query rows are computed.

    Returns:
      out [n, Hq, Dv] float64 and lse [Hq, n] float64, where n = Nt or len(rows).
    """
    if window < 0:
        raise ValueError("window must be >= 0")
    K, Vv = _f64(k), _f64(v)
    cu = _i64(cu_seqlens)
    Nt, Hq, Dqk = q.shape
    Hkv, Dv = K.shape[1], Vv.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    sig = np.full(Hq, -np.inf) if sinks is None else _f64(sinks).reshape(Hq)

    if rows is None:
        rows = np.arange(Nt)
        Q = _f64(q)                       # [n, Hq, Dqk], row t = token t
    else:
        rows = _i64(rows).reshape(-1)
        if hasattr(q, "detach"):
            import torch

            Q = _f64(q[torch.as_tensor(rows, device=q.device)])
        else:
            Q = _f64(np.asarray(q)[rows])
    n = rows.shape[0]
    out = np.zeros((n, Hq, Dv))
    lse = np.full((Hq, n), -np.inf)
    if n == 0:
        return out, lse
    seq_of = np.searchsorted(cu, rows, side="right") - 1

    jobs = []
    for s in np.unique(seq_of):
        b0, b1 = int(cu[s]), int(cu[s + 1])
        sel = np.nonzero(seq_of == s)[0]
        qpos = rows[sel] - b0
        kpos = np.arange(b1 - b0)
        for h in range(Hq):
            jobs.append((sel, qpos, b0, b1, h, kpos))

    def run(job):
        sel, qpos, b0, b1, h, kpos = job
        g = h // G
        o, l = _one_head(Q[sel, h, :], K[b0:b1, g, :], Vv[b0:b1, g, :],
                         qpos, kpos, window, sig[h], scale)
        return sel, h, o, l

    nthreads = threads or len(os.sched_getaffinity(0))
    # one BLAS thread per worker: the pool over (sequence, head) jobs uses the cores
    with _blas_threads(1), ThreadPoolExecutor(max_workers=nthreads) as ex:
        for sel, h, o, l in ex.map(run, jobs):
            out[sel, h, :] = o * v_scale
            lse[h, sel] = l
    return out, lse


def ring_slot_position(slot, L, C):
    """Absolute token position held by ring slot ``slot``.

    A ring cache of ``C`` slots keeps token ``p`` in slot ``p mod C``; with
    ``L`` tokens written so far (the current one included) the valid slots
    are ``slot < min(L, C)`` and hold the most recent ``min(L, C)`` tokens.
    """
    slot = np.asarray(slot)
    if L <= C:
        return slot.copy()
    return (L - 1) - np.mod((L - 1) - slot, C)


def decode(q, k_cache, v_cache, seqlens, window, sinks, ring=None, scale=None,
           v_scale=1.0, batch_index=None):
    """One decode step per sequence, float64, written from the definition.

    Args:
      q: [B, Hq, Dqk] the current token's queries (post-RoPE).
      k_cache: [B, C, Hkv, Dqk]; v_cache: [B, C, Hkv, Dv].
      seqlens: [B] tokens so far *including* the current one, whose K/V are
        already in the cache; the query sits at position ``L - 1``.
      window: 0 = global; >= 1 = query plus previous ``window - 1`` keys.
      ring: cache is a ring of ``C`` slots (token p in slot p mod C).  Default:
        ``window > 0 and C == window``.  Otherwise slot = position (linear).
      batch_index: optional subset of sequences to compute.

    Returns:
      out [n, Hq, Dv] and lse [n, Hq] (float64), n = B or len(batch_index).
    """
    if window < 0:
        raise ValueError("window must be >= 0")
    B, Hq, Dqk = q.shape
    C, Hkv = k_cache.shape[1], k_cache.shape[2]
    Dv = v_cache.shape[3]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    if ring is None:
        ring = window > 0 and C == window
    sig = np.full(Hq, -np.inf) if sinks is None else _f64(sinks).reshape(Hq)
    Ls = _i64(seqlens).reshape(-1)
    idx = np.arange(B) if batch_index is None else _i64(batch_index).reshape(-1)

    out = np.zeros((len(idx), Hq, Dv))
    lse = np.full((len(idx), Hq), -np.inf)
    for n, b in enumerate(idx):
        L = int(Ls[b])
        nvalid = min(L, C)
        if L < 0 or (not ring and L > C):
            raise ValueError("seqlen outside the cache")
        slots = np.arange(nvalid)
        pos = ring_slot_position(slots, L, C) if ring else slots
        keep = visible(L - 1, pos, window)
        slots = slots[keep]
        qb = _f64(q[b])                                  # [Hq, Dqk]
        s0 = int(slots[0]) if len(slots) else 0
        s1 = int(slots[-1]) + 1 if len(slots) else 0
        for g in range(Hkv):
            Kg = _f64(k_cache[b, s0:s1, g, :])[slots - s0] if len(slots) else np.zeros((0, Dqk))
            Vg = _f64(v_cache[b, s0:s1, g, :])[slots - s0] if len(slots) else np.zeros((0, Dv))
            for h in range(g * G, (g + 1) * G):
                S = scale * (Kg @ qb[h])
                m = max(sig[h], S.max() if len(S) else -np.inf)
                if not np.isfinite(m):
                    continue  # nothing visible and no sink: out = 0, lse = -inf
                e = np.exp(S - m)
                Z = e.sum() + math.exp(sig[h] - m)
                out[n, h] = v_scale * (e @ Vg) / Z
                lse[n, h] = m + math.log(Z)
    return out, lse
