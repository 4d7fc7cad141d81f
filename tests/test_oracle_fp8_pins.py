"""Pins for the oracle's FP8 (e4m3) KV-cache decode, against things other than itself.

CPU only.  The e4m3 decoder is pinned to torch's float8_e4m3fn conversion (a
library routine) on all 256 codes and to values fixed by the format's
definition; decode_fp8 is pinned to the plain decode over caches dequantised
by torch, and to the linearity of the two per-head scales.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle.fp8 import decode_fp8, e4m3_to_float
from workloads import decode_inputs_fp8


def test_e4m3_decoder_matches_torch_on_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine = e4m3_to_float(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[~np.isnan(mine)], ref[~np.isnan(ref)])
    # signed zeros too
    assert np.signbit(mine[0x80]) and not np.signbit(mine[0x00])


@pytest.mark.parametrize("code,value", [
    (0x38, 1.0),            # e = 7, m = 0
    (0x3C, 1.5),            # e = 7, m = 4
    (0x40, 2.0),            # e = 8
    (0xC0, -2.0),
    (0x7E, 448.0),          # largest finite: e = 15, m = 6
    (0xFE, -448.0),
    (0x08, 2.0 ** -6),      # smallest normal
    (0x01, 2.0 ** -9),      # smallest subnormal: (1/8) 2^-6
    (0x07, 7 * 2.0 ** -9),  # largest subnormal
    (0x00, 0.0),
])
def test_e4m3_format_values(code, value):
    assert e4m3_to_float(np.array([code], dtype=np.uint8))[0] == value


def test_e4m3_nan_codes():
    v = e4m3_to_float(np.array([0x7F, 0xFF, 0x7E, 0x78], dtype=np.uint8))
    assert np.isnan(v[0]) and np.isnan(v[1]) and v[2] == 448.0 and v[3] == 256.0


def _dequant_torch(codes, scale):
    return codes.view(torch.float8_e4m3fn).to(torch.float64) * scale.to(torch.float64).view(1, 1, -1, 1)


@pytest.mark.parametrize("window,cap,lengths", [
    (0, 40, [1, 17, 40]),        # global, linear
    (3, 40, [2, 3, 33]),         # window on a linear cache
    (5, 5, [1, 4, 5, 6, 13]),    # ring of 5 slots (L <= C and L > C)
])
def test_decode_fp8_equals_decode_on_library_dequantised_caches(window, cap, lengths):
    x = decode_inputs_fp8(lengths, cap, window, hq=4, hkv=2, dqk=8, dv=4, seed=5, poison=False)
    kd = _dequant_torch(x.k_codes, x.k_scale)
    vd = _dequant_torch(x.v_codes, x.v_scale_kv)
    ref = oracle.decode(x.q, kd, vd, x.seqlens, window, x.sinks)
    got = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, window, x.sinks)
    np.testing.assert_allclose(got[0], ref[0], atol=1e-13, rtol=0)
    np.testing.assert_allclose(got[1], ref[1], atol=1e-13, rtol=0)


def test_decode_fp8_ignores_poisoned_slots():
    x = decode_inputs_fp8([3, 7], 10, 0, hq=2, hkv=1, dqk=8, dv=4, seed=2, poison=True)
    assert int(x.k_codes[0, 5, 0, 0]) == 0x7F
    out, lse = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, 0, x.sinks)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def test_fp8_scales_are_linear():
    """k_scale multiplies every score like the softmax scale; v_scale_kv multiplies the output."""
    x = decode_inputs_fp8([9, 20], 24, 0, hq=4, hkv=2, dqk=8, dv=4, seed=9)
    c = 1.75
    base_scale = 1.0 / np.sqrt(8.0)
    a = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale.double() * c, x.v_scale_kv, x.seqlens, 0, x.sinks,
                   scale=base_scale)
    b = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, 0, x.sinks,
                   scale=base_scale * c)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], atol=1e-13)
    u = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv.double() * c, x.seqlens, 0, x.sinks)
    w = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, 0, x.sinks,
                   v_scale=c)
    np.testing.assert_allclose(u[0], w[0], atol=1e-13)
    np.testing.assert_allclose(u[1], w[1], atol=1e-13)


def test_fp8_scale_pin_detects_a_wrong_head_mapping():
    """Applying head 0's scale to every head changes the result (the pin above has teeth)."""
    x = decode_inputs_fp8([12], 16, 0, hq=4, hkv=2, dqk=8, dv=4, seed=3)
    good = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, 0, x.sinks)
    flat = x.k_scale[:1].repeat(2)
    bad = decode_fp8(x.q, x.k_codes, x.v_codes, flat, x.v_scale_kv, x.seqlens, 0, x.sinks)
    assert np.abs(good[1] - bad[1]).max() > 1e-6
