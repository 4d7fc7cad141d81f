"""Pins for the oracle's context-parallel merge, against the single decode.

CPU only.  Splitting a cache's keys into disjoint parts, decoding each part
without the sink and merging must reproduce the decode over all keys with the
sink (any split, empty parts included); a merge that forgot the sink or
weighted parts equally fails.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle.merge import merge
from workloads import decode_inputs


def _parts(x, cuts):
    """Decode each slice [cuts[i], cuts[i+1]) of every sequence's keys without the sink."""
    B = x.q.shape[0]
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        lens = []
        ks = torch.zeros((B, max(1, b - a)) + tuple(x.k_cache.shape[2:]), dtype=x.k_cache.dtype)
        vs = torch.zeros((B, max(1, b - a)) + tuple(x.v_cache.shape[2:]), dtype=x.v_cache.dtype)
        for i, L in enumerate(x.seqlens.tolist()):
            n = max(0, min(L, b) - a)
            lens.append(n)
            if n:
                ks[i, :n] = x.k_cache[i, a:a + n]
                vs[i, :n] = x.v_cache[i, a:a + n]
        o, l = oracle.decode(x.q, ks, vs, lens, 0, None, ring=False)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("cuts", [[0, 40], [0, 13, 40], [0, 1, 2, 39, 40], [0, 20, 20, 40]])
@pytest.mark.parametrize("sinks", [True, False])
def test_merge_of_parts_equals_full_decode(cuts, sinks):
    x = decode_inputs([1, 7, 25, 40], 40, 0, hq=4, hkv=2, dqk=8, dv=4, seed=11, sinks=sinks,
                      poison=False)
    po, pl = _parts(x, cuts)
    got = merge(po, pl, x.sinks, v_scale=0.7)
    ref = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks, v_scale=0.7)
    np.testing.assert_allclose(got[0], ref[0], atol=1e-13)
    np.testing.assert_allclose(got[1], ref[1], atol=1e-13)


def test_merge_pin_has_teeth():
    x = decode_inputs([30, 40], 40, 0, hq=2, hkv=1, dqk=8, dv=4, seed=12, poison=False)
    po, pl = _parts(x, [0, 10, 40])
    ref = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    no_sink = merge(po, pl, None)
    equal_w = (po.mean(axis=0), pl.max(axis=0))
    assert np.abs(no_sink[0] - ref[0]).max() > 1e-6
    assert np.abs(equal_w[0] - ref[0]).max() > 1e-6


def test_empty_part_output_is_ignored():
    """An empty part (lse -inf) may carry any output values, NaN included."""
    rng = np.random.default_rng(3)
    po = rng.standard_normal((3, 2, 2, 4))
    pl = rng.standard_normal((3, 2, 2))
    pl[1, 0] = -np.inf
    clean = merge(po, pl, None)
    po[1, 0] = np.nan
    dirty = merge(po, pl, None)
    np.testing.assert_array_equal(dirty[0], clean[0])
    np.testing.assert_array_equal(dirty[1], clean[1])


def test_all_parts_empty():
    po = np.zeros((2, 1, 3, 4))
    pl = np.full((2, 1, 3), -np.inf)
    out, lse = merge(po, pl, None)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    s = torch.tensor([0.5, -1.0, 2.0])
    out, lse = merge(po, pl, s)
    assert np.all(out == 0)
    np.testing.assert_allclose(lse[0], s.double().numpy())
