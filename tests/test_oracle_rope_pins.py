"""Pins for the oracle's rotary embedding and decode-step cache append.

CPU only.  RoPE is pinned to closed forms (a 2-dimension rotation, hand
values of the rotate-half pairing and the frequencies) and to the properties
that define it (identity at position 0, norm-preserving pairs, rotations that
compose by adding positions, dot products that depend only on the position
difference); the append is pinned to the slot arithmetic and to the ring
reading of the decode.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle.rope import append_slot, rope, rope_angles, rope_append
from workloads import decode_inputs


def _x(shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def test_position_zero_is_identity():
    x = _x((4, 3, 16))
    np.testing.assert_array_equal(rope(x, np.zeros(4), 10000.0), x)


def test_pairs_keep_their_norm():
    x = _x((5, 2, 12), 1)
    y = rope(x, np.array([1, 7, 100, 4096, 262143]), 10000.0)
    h = 6
    nx = x[..., :h] ** 2 + x[..., h:] ** 2
    ny = y[..., :h] ** 2 + y[..., h:] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


def test_rotations_compose_by_adding_positions():
    x = _x((3, 16), 2)
    p = np.array([3, 50, 1000])
    s = np.array([9, 1, 77])
    np.testing.assert_allclose(rope(rope(x, p, 500.0), s, 500.0), rope(x, p + s, 500.0), atol=1e-11)


def test_dot_products_depend_on_the_position_difference_only():
    q, k = _x((1, 32), 3), _x((1, 32), 4)
    d0 = float((rope(q, [10], 10000.0) @ rope(k, [3], 10000.0).T)[0, 0])
    d1 = float((rope(q, [1010], 10000.0) @ rope(k, [1003], 10000.0).T)[0, 0])
    d2 = float((rope(q, [7], 10000.0) @ rope(k, [0], 10000.0).T)[0, 0])
    assert abs(d0 - d1) < 1e-10 and abs(d0 - d2) < 1e-10


def test_two_dimensions_is_a_plane_rotation():
    x = np.array([[0.6, -1.3]])
    for p in (0, 1, 2.5, 17):
        a = float(p)  # i = 0: frequency theta^0 = 1
        want = [0.6 * math.cos(a) + 1.3 * math.sin(a), -1.3 * math.cos(a) + 0.6 * math.sin(a)]
        np.testing.assert_allclose(rope(x, [p], 10000.0)[0], want, atol=1e-15)


def test_rotate_half_pairing_and_frequencies():
    # d = 4: pairs (0, 2) and (1, 3); frequencies 1 and theta^(-1/2)
    np.testing.assert_allclose(rope_angles([3], 10000.0, 4)[0], [3.0, 0.03], rtol=1e-15)
    e0 = np.array([[1.0, 0.0, 0.0, 0.0]])
    y = rope(e0, [1], 10000.0)[0]
    np.testing.assert_allclose(y, [math.cos(1), 0.0, math.sin(1), 0.0], atol=1e-15)
    e1 = np.array([[0.0, 1.0, 0.0, 0.0]])
    y = rope(e1, [1], 10000.0)[0]
    np.testing.assert_allclose(y, [0.0, math.cos(0.01), 0.0, math.sin(0.01)], atol=1e-15)


def test_partial_rotary_leaves_the_tail():
    x = _x((2, 3, 20), 5)
    y = rope(x, [4, 9], 10000.0, rotary_dim=8)
    np.testing.assert_array_equal(y[..., 8:], x[..., 8:])
    np.testing.assert_allclose(y[..., :8], rope(x[..., :8], [4, 9], 10000.0), atol=0)


def test_append_slot_arithmetic():
    assert append_slot(1, 10, False) == 0
    assert append_slot(10, 10, False) == 9
    with pytest.raises(ValueError):
        append_slot(11, 10, False)
    assert append_slot(129, 129, True) == 128
    assert append_slot(130, 129, True) == 0
    assert append_slot(1000, 129, True) == 999 % 129


@pytest.mark.parametrize("window,cap,lengths", [(0, 16, [1, 9, 16]), (5, 5, [1, 5, 6, 12])])
def test_append_writes_one_slot(window, cap, lengths):
    x = decode_inputs(lengths, cap, window, hq=4, hkv=2, dqk=8, dv=4, seed=6, poison=False)
    rng = np.random.default_rng(7)
    kn = rng.standard_normal((len(lengths), 2, 8))
    vn = rng.standard_normal((len(lengths), 2, 4))
    q_rot, kc, vc = rope_append(x.q, kn, vn, x.k_cache, x.v_cache, x.seqlens, window, 1000.0)
    k0 = x.k_cache.double().numpy()
    v0 = x.v_cache.double().numpy()
    for b, L in enumerate(lengths):
        slot = append_slot(L, cap, window > 0 and cap == window)
        mask = np.ones(cap, bool)
        mask[slot] = False
        np.testing.assert_array_equal(kc[b, mask], k0[b, mask])
        np.testing.assert_array_equal(vc[b, mask], v0[b, mask])
        np.testing.assert_allclose(kc[b, slot], rope(kn[b:b + 1], [L - 1], 1000.0)[0], atol=0)
        np.testing.assert_array_equal(vc[b, slot], vn[b])
    np.testing.assert_allclose(q_rot, rope(x.q, np.array(lengths) - 1, 1000.0), atol=0)


def test_ring_append_then_decode_equals_linear_window():
    """Appending token after token into a 5-slot ring and decoding equals the linear cache
    with window 5 (both hold the same rotated keys)."""
    W, T = 5, 13
    rng = np.random.default_rng(8)
    qs = rng.standard_normal((T, 2, 8))
    ks = rng.standard_normal((T, 1, 8))
    vs = rng.standard_normal((T, 1, 4))
    ring_k = np.zeros((1, W, 1, 8))
    ring_v = np.zeros((1, W, 1, 4))
    lin_k = np.zeros((1, T, 1, 8))
    lin_v = np.zeros((1, T, 1, 4))
    sinks = torch.tensor([0.3, -1.0])
    for t in range(T):
        L = np.array([t + 1])
        q_r, ring_k, ring_v = rope_append(qs[t:t + 1], ks[t:t + 1], vs[t:t + 1], ring_k, ring_v, L, W, 100.0)
        _, lin_k, lin_v = rope_append(qs[t:t + 1], ks[t:t + 1], vs[t:t + 1], lin_k, lin_v, L, W, 100.0)
        a = oracle.decode(q_r, ring_k, ring_v, L, W, sinks)
        b = oracle.decode(q_r, lin_k, lin_v, L, W, sinks, ring=False)
        np.testing.assert_allclose(a[0], b[0], atol=1e-13)
        np.testing.assert_allclose(a[1], b[1], atol=1e-13)
