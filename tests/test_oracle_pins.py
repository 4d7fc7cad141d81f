"""Pins for the fp64 oracle, against things other than itself.

CPU only.  Each test names what it pins the oracle to:
brute force, a closed form, a library special case (torch SDPA), an
invariant, or a constant the MiMo-V2-Flash documentation prints.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from workloads import cu_seqlens_of, decode_inputs, prefill_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "config_constants.json")


def _small(lengths, hq=4, hkv=2, dqk=8, dv=4, seed=0, sinks=True):
    return prefill_inputs(lengths, hq=hq, hkv=hkv, dqk=dqk, dv=dv, seed=seed, sinks=sinks)


# --------------------------------------------------------------------------
# brute force


@pytest.mark.parametrize("window", [0, 1, 2, 3, 5, 100])
@pytest.mark.parametrize("sinks", [True, False])
def test_vectorised_matches_scalar_brute_force(window, sinks):
    x = _small([0, 1, 5, 17, 9], sinks=sinks, seed=window + 11)
    scale = 1.0 / math.sqrt(8)
    out, lse = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, scale=scale)
    bo, bl = brute.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, scale)
    np.testing.assert_allclose(out, np.array(bo), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-12)


def test_row_subset_matches_full():
    x = _small([7, 300, 40], seed=3)
    out, lse = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens)
    rows = np.array([0, 6, 7, 8, 100, 306, 307, 346])
    o2, l2 = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens, rows=rows)
    np.testing.assert_allclose(o2, out[rows], atol=1e-13)
    np.testing.assert_allclose(l2, lse[:, rows], atol=1e-13)


# --------------------------------------------------------------------------
# windows


def test_window_at_least_T_is_global():
    x = _small([33, 20], seed=5)
    g = oracle.prefill(x.q, x.k, x.v, x.sinks, 0, x.cu_seqlens)
    for W in (33, 34, 1000):
        w = oracle.prefill(x.q, x.k, x.v, x.sinks, W, x.cu_seqlens)
        np.testing.assert_array_equal(w[0], g[0])
        np.testing.assert_array_equal(w[1], g[1])


def test_window_one_closed_form():
    """W=1: only the token itself -> out_i = e^s/(e^s + e^sigma) * v_i, s = <q_i,k_i>/sqrt(192)."""
    x = prefill_inputs([19], hq=4, hkv=1, seed=9)
    out, lse = oracle.prefill(x.q, x.k, x.v, x.sinks, 1, x.cu_seqlens)
    q, k, v = (t.double().numpy() for t in (x.q, x.k, x.v))
    sg = x.sinks.double().numpy()
    for i in range(19):
        for h in range(4):
            s = float(q[i, h] @ k[i, 0]) / math.sqrt(192.0)
            p = math.exp(s) / (math.exp(s) + math.exp(sg[h]))
            np.testing.assert_allclose(out[i, h], p * v[i, 0], rtol=1e-12, atol=1e-14)
            assert abs(lse[h, i] - math.log(math.exp(s) + math.exp(sg[h]))) < 1e-12


def test_window_one_pin_detects_wrong_scale():
    """A planted mistake (scale 1/sqrt(Dv) instead of 1/sqrt(Dqk)) fails the W=1 pin."""
    x = prefill_inputs([8], hq=2, hkv=1, seed=9)
    good, _ = oracle.prefill(x.q, x.k, x.v, x.sinks, 1, x.cu_seqlens)
    bad, _ = oracle.prefill(x.q, x.k, x.v, x.sinks, 1, x.cu_seqlens, scale=1 / math.sqrt(128))
    assert np.abs(good - bad).max() > 1e-3


# --------------------------------------------------------------------------
# sink


def _sdpa_reference(x, window, scale):
    """torch CPU float64 SDPA with an explicit boolean mask and repeated K/V heads."""
    outs = []
    cu = x.cu_seqlens.tolist()
    hq, hkv = x.q.shape[1], x.k.shape[1]
    for s in range(len(cu) - 1):
        b0, b1 = cu[s], cu[s + 1]
        T = b1 - b0
        if T == 0:
            continue
        q = x.q[b0:b1].double().transpose(0, 1)  # [H, T, D]
        k = x.k[b0:b1].double().transpose(0, 1).repeat_interleave(hq // hkv, dim=0)
        v = x.v[b0:b1].double().transpose(0, 1).repeat_interleave(hq // hkv, dim=0)
        i = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        mask = (i - j >= 0)
        if window > 0:
            mask &= (i - j <= window - 1)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
        outs.append(o.transpose(0, 1))
    return torch.cat(outs).numpy()


@pytest.mark.parametrize("window", [0, 1, 4, 129])
def test_no_sink_is_plain_softmax_sdpa(window):
    x = prefill_inputs([1, 37, 150], hq=8, hkv=2, dqk=16, dv=8, seed=21, sinks=False)
    scale = 1 / math.sqrt(16)
    out, _ = oracle.prefill(x.q, x.k, x.v, None, window, x.cu_seqlens, scale=scale)
    np.testing.assert_allclose(out, _sdpa_reference(x, window, scale), atol=1e-12)


def test_sink_is_a_zero_value_virtual_key():
    """Appending a key with score sigma (q.k = sigma/s) and value 0 equals the sink."""
    x = prefill_inputs([12], hq=2, hkv=1, dqk=4, dv=3, seed=4)
    s = 1 / math.sqrt(4)
    out, lse = oracle.prefill(x.q, x.k, x.v, x.sinks, 0, x.cu_seqlens, scale=s)
    q, k, v = (t.double().numpy() for t in (x.q, x.k, x.v))
    for i in range(12):
        for h in range(2):
            sc = [s * float(q[i, h] @ k[j, 0]) for j in range(i + 1)] + [float(x.sinks[h])]
            w = np.exp(np.array(sc) - max(sc))
            w /= w.sum()
            ref = (w[:-1, None] * v[: i + 1, 0]).sum(0)
            np.testing.assert_allclose(out[i, h], ref, atol=1e-13)


def test_constant_values_give_one_minus_sink_mass():
    """V = c everywhere -> out = c * (1 - exp(sigma - lse)): pins lse and the sink together."""
    x = prefill_inputs([50, 3], hq=4, hkv=2, dqk=8, dv=4, seed=2)
    c = 0.625
    v = torch.full_like(x.v, c)
    out, lse = oracle.prefill(x.q, x.k, v, x.sinks, 7, x.cu_seqlens)
    sink_mass = np.exp(x.sinks.double().numpy()[:, None] - lse)  # [H, Nt]
    expect = np.broadcast_to(c * (1 - sink_mass.T)[:, :, None], out.shape)
    np.testing.assert_allclose(out, expect, atol=1e-13)


@pytest.mark.parametrize("window", [0, 5])
def test_zero_query_closed_form(window):
    """q = 0 -> all n visible scores are 0: out = sum v / (n + e^sigma), lse = ln(n + e^sigma)."""
    x = prefill_inputs([23], hq=2, hkv=1, dqk=8, dv=4, seed=8)
    q = torch.zeros_like(x.q)
    out, lse = oracle.prefill(q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    v = x.v.double().numpy()[:, 0]
    for i in range(23):
        lo = 0 if window == 0 else max(0, i - window + 1)
        n = i + 1 - lo
        for h in range(2):
            es = math.exp(float(x.sinks[h]))
            np.testing.assert_allclose(out[i, h], v[lo:i + 1].sum(0) / (n + es), atol=1e-13)
            assert abs(lse[h, i] - math.log(n + es)) < 1e-13


def test_probability_mass_sums_to_one():
    x = prefill_inputs([40], hq=2, hkv=1, dqk=8, dv=4, seed=12)
    s = 1 / math.sqrt(8)
    out, lse = oracle.prefill(x.q, x.k, x.v, x.sinks, 9, x.cu_seqlens, scale=s)
    q, k = x.q.double().numpy(), x.k.double().numpy()
    for i in range(40):
        for h in range(2):
            j = np.arange(max(0, i - 8), i + 1)
            S = s * (k[j, 0] @ q[i, h])
            total = np.exp(S - lse[h, i]).sum() + math.exp(float(x.sinks[h]) - lse[h, i])
            assert abs(total - 1.0) < 1e-13


def test_linearity_in_v():
    x = _small([30], seed=13)
    a, la = oracle.prefill(x.q, x.k, x.v, x.sinks, 4, x.cu_seqlens)
    b, lb = oracle.prefill(x.q, x.k, x.v, x.sinks, 4, x.cu_seqlens, v_scale=0.707)
    np.testing.assert_allclose(b, 0.707 * a, atol=1e-14)
    np.testing.assert_array_equal(la, lb)


def test_gqa_grouping_is_consecutive():
    """Heads 0..G-1 read KV head 0: zeroing KV head 1 changes only heads G..2G-1."""
    x = prefill_inputs([16], hq=4, hkv=2, dqk=8, dv=4, seed=14)
    a, _ = oracle.prefill(x.q, x.k, x.v, x.sinks, 0, x.cu_seqlens)
    v2 = x.v.clone()
    v2[:, 1] = 0
    b, _ = oracle.prefill(x.q, x.k, v2, x.sinks, 0, x.cu_seqlens)
    np.testing.assert_array_equal(a[:, :2], b[:, :2])
    assert np.abs(b[:, 2:]).max() == 0.0


# --------------------------------------------------------------------------
# decode


@pytest.mark.parametrize("window", [0, 3, 129])
def test_decode_equals_last_prefill_row(window):
    T = 140
    x = prefill_inputs([T], hq=4, hkv=2, dqk=8, dv=4, seed=31)
    out, lse = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    for L in (1, 2, 100, 140):
        kc = x.k[:L].unsqueeze(0)
        vc = x.v[:L].unsqueeze(0)
        q = x.q[L - 1].unsqueeze(0)
        od, ld = oracle.decode(q, kc, vc, [L], window, x.sinks, ring=False)
        np.testing.assert_allclose(od[0], out[L - 1], atol=1e-13)
        np.testing.assert_allclose(ld[0], lse[:, L - 1], atol=1e-13)


def _to_ring(k, L, C):
    """Place the last min(L, C) of L tokens into ring slots p mod C."""
    ring = torch.full((C,) + tuple(k.shape[1:]), float("nan"), dtype=k.dtype)
    for p in range(max(0, L - C), L):
        ring[p % C] = k[p]
    return ring


@pytest.mark.parametrize("L", [1, 5, 129, 130, 300, 517])
def test_ring_equals_linear_cache_with_window(L):
    C = W = 129
    x = prefill_inputs([L], hq=4, hkv=2, dqk=8, dv=4, seed=L)
    lin = oracle.decode(x.q[L - 1:L], x.k[:L][None], x.v[:L][None], [L], W, x.sinks, ring=False)
    kr, vr = _to_ring(x.k[:L], L, C), _to_ring(x.v[:L], L, C)
    rng = oracle.decode(x.q[L - 1:L], kr[None], vr[None], [L], W, x.sinks, ring=True)
    np.testing.assert_allclose(rng[0], lin[0], atol=1e-13)
    np.testing.assert_allclose(rng[1], lin[1], atol=1e-13)


def test_ring_slot_positions():
    C = 5
    # L <= C: slot s holds position s
    assert list(oracle.ring_slot_position(np.arange(3), 3, C)) == [0, 1, 2]
    # L = 12: positions 7..11 live in slots 7%5=2, 3, 4, 0, 1
    pos = oracle.ring_slot_position(np.arange(5), 12, C)
    assert list(pos) == [10, 11, 7, 8, 9]
    assert all(p % C == s for s, p in enumerate(pos))


def test_decode_empty_sequence_gives_zero_and_sink_lse():
    x = decode_inputs([0, 3], 8, 0, hq=2, hkv=1, dqk=8, dv=4, seed=1, poison=False)
    out, lse = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    assert np.all(out[0] == 0)
    np.testing.assert_allclose(lse[0], x.sinks.double().numpy(), atol=0)
    out2, lse2 = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, None)
    assert np.all(out2[0] == 0) and np.all(np.isneginf(lse2[0]))


def test_decode_ignores_poisoned_slots():
    x = decode_inputs([3, 7], 10, 0, hq=2, hkv=1, dqk=8, dv=4, seed=2, poison=True)
    out, lse = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


# --------------------------------------------------------------------------
# constants the documentation prints


def test_attention_value_scale_constant():
    c = json.load(open(GOLDEN))
    val = math.sqrt(c["hidden_size"] / (c["num_attention_heads"] * c["v_head_dim"]))
    assert abs(val - 0.70710678) < 1e-8
    assert abs(val - c["attention_value_scale"]) < 5e-4


def test_kv_cache_reduction_about_six():
    """48 layers at 5:1 -> 8 global + 40 SWA; ratio 48L / (8L + 40 min(L, 129))."""
    c = json.load(open(GOLDEN))
    n = c["num_hidden_layers"]
    swa, ga = c["swa_to_global_ratio"]
    n_ga = n * ga // (swa + ga)
    n_swa = n - n_ga
    assert (n_ga, n_swa) == (8, 40)
    W = c["sliding_window"]

    def ratio(L):
        return n * L / (n_ga * L + n_swa * min(L, W))

    assert abs(ratio(c["context_window_tokens"]) - 5.985) < 1e-3
    assert abs(ratio(32768) - 5.884) < 1e-3
    assert 5.5 < ratio(c["context_window_tokens"]) < 6.0   # "about 6x"
    # the prose's 128-token window is W - 1 previous keys
    assert W - 1 == c["prose_window_tokens"]
