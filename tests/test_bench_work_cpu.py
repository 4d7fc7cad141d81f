"""The benchmark's work model (the numerators of every roofline fraction), CPU only.

Visible pairs are checked against brute force over the mask definition (query
i sees key j iff 0 <= i - j and, with a window W > 0, i - j <= W - 1); the
FLOP and byte counts against the per-unit figures the model's head shape
fixes (MiMoV2FlashConfig: 64 query / 4 key-value heads, head_dim 192,
v_head_dim 128): 2*192 + 2*128 = 640 flop per (visible pair, query head),
K+V of 4 heads = 2560 bytes per cached token, and per prefill token
q + k + v read once and out (bf16) + lse written once.
"""

import numpy as np
import pytest

import bench
import workloads as W


def brute_pairs(T, window):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    d = i - j
    vis = d >= 0
    if window > 0:
        vis &= d <= window - 1
    return int(vis.sum())


@pytest.mark.parametrize("T,window", [(1, 0), (7, 0), (300, 129), (128, 129), (129, 129), (130, 129),
                                      (4095, 129), (4096, 129), (5000, 129), (5000, 1), (4500, 0),
                                      (200, 500)])
def test_visible_pairs_match_brute_force(T, window):
    assert bench.visible_pairs(T, window) == brute_pairs(T, window)


def test_per_unit_figures():
    assert bench.FLOP_PER_PAIR == 640
    assert bench.KV_BYTES_PER_TOKEN == 2560


def test_prefill_work_at_the_benchmark_sizes():
    # sliding window 129 at T=32768: 129*130/2 + (32768-129)*129 visible pairs
    f, b = bench.prefill_work(32768, 129)
    assert f == 640 * 64 * 4_218_816
    # 64*192*2 + 4*(192+128)*2 + 64*128*2 + 64*4 = 43,776 bytes per token
    assert b == 32768 * 43_776 == 1_434_451_968
    f, b = bench.prefill_work(32768, 0)
    assert f == 640 * 64 * (32768 * 32769 // 2)
    assert round(f / 1e13, 3) == 2.199


def test_decode_work_at_the_benchmark_sizes():
    lengths = W.decode_b64_lengths(0)
    assert len(lengths) == 64 and min(lengths) >= 1024 and max(lengths) <= 262144
    total = int(sum(lengths))
    f, b = bench.decode_work(lengths, 0, W.DECODE_GA_CAPACITY)
    assert f == 640 * 64 * total
    # K+V bytes of every visible key + q read and out / lse written per (sequence, head)
    assert b == total * 2560 + 64 * 64 * (192 * 2 + 128 * 2 + 4)
    # a 129-slot ring holds min(L, 129) keys per sequence
    f, b = bench.decode_work(lengths, 129, 129)
    assert f == 640 * 64 * 64 * 129
    # e4m3 caches: one byte per element plus the per-KV-head K and V scales
    _, b8 = bench.decode_fp8_work(lengths, 0, W.DECODE_GA_CAPACITY)
    assert b8 == total * 1280 + 64 * 64 * (192 * 2 + 128 * 2 + 4) + 2 * 4 * 4


def test_varlen_stack_work():
    """Config 5: 16 packed sequences ~U[512, 8192] (Nt = 70,172), five window-129
    layers and one global layer: per-layer work is the sum over sequences."""
    lengths = W.varlen_stack_lengths(0)
    assert len(lengths) == 16 and sum(lengths) == 70172
    f_swa, b_swa = bench.varlen_prefill_work(lengths, 129)
    f_ga, b_ga = bench.varlen_prefill_work(lengths, 0)
    assert f_swa == 640 * 64 * sum(brute_pairs(L, 129) for L in lengths[:2]) + 640 * 64 * sum(
        bench.visible_pairs(L, 129) for L in lengths[2:])
    assert f_ga == 640 * 64 * sum(L * (L + 1) // 2 for L in lengths)
    assert b_swa == b_ga == 70172 * 43_776
    assert round((5 * f_swa + f_ga) / 1e12, 2) == 9.99
