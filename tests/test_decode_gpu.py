"""Decode kernels (split-KV mma.sync + combine) vs the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def run(x, out_dtype=torch.float32, v_scale=1.0):
    q, k, v, sl = (t.to("cuda") for t in (x.q, x.k_cache, x.v_cache, x.seqlens))
    s = None if x.sinks is None else x.sinks.to("cuda")
    out, lse = mimo.mimo_attn_decode(q, k, v, sl, x.window, s, out_dtype=out_dtype, v_scale=v_scale)
    mimo.mimo_attn_device_status()
    return out, lse


@pytest.mark.parametrize("window,capacity", [(0, 1024), (129, 1024), (129, 129), (1, 16), (0, 8192)])
@pytest.mark.parametrize("sinks", [True, False])
def test_small_batches(window, capacity, sinks):
    lengths = [1, 5, 64, 65, 130, 1000, 129, 128] if capacity >= 1000 else [1, 5, 16, 200, 129, 3]
    if capacity < 1000 and window == 1:
        lengths = [1, 2, 16, 9]
    if window == 0 or window != capacity:
        lengths = [min(L, capacity) for L in lengths]
    x = W.decode_inputs(lengths, capacity, window, hq=8, hkv=2, seed=capacity + window, sinks=sinks)
    out, lse = run(x)
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, window, x.sinks)
    P.check(out, ro, lse, rl, what=f"W={window} C={capacity}")


def test_empty_sequence():
    x = W.decode_inputs([0, 7], 64, 0, hq=4, hkv=1, seed=3)
    out, lse = run(x)
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    P.check(out, ro, lse, rl, what="empty")


def test_model_heads_bf16_out():
    x = W.decode_inputs([3000, 17, 4097], 8192, 0, seed=9)
    out, lse = run(x, torch.bfloat16)
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    P.check(out, ro, lse, rl, what="64/4 heads")


def test_split_count_does_not_change_the_result():
    """Same data in caches of different capacity -> different split plans."""
    lengths = [5000, 300, 70]
    a = W.decode_inputs(lengths, 8192, 0, seed=12, poison=False)
    outs = []
    for cap in (8192, 65536, 5000):
        k = torch.zeros((3, cap, 4, 192), dtype=torch.bfloat16)
        v = torch.zeros((3, cap, 4, 128), dtype=torch.bfloat16)
        n = min(cap, 8192)
        k[:, :n] = a.k_cache[:, :n]
        v[:, :n] = a.v_cache[:, :n]
        x = W.DecodeInputs(a.q, k, v, a.seqlens, a.sinks, 0, cap)
        outs.append(run(x)[0])
    ro, _ = oracle.decode(a.q, a.k_cache, a.v_cache, a.seqlens, 0, a.sinks)
    for o in outs:
        P.check(o, ro, what="split plan")


def test_decode_equals_last_prefill_row():
    T = 700
    x = W.prefill_inputs([T], hq=64, hkv=4, seed=21)
    po, pl = mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.sinks.cuda(), 0,
                                    x.cu_seqlens.cuda(), T, out_dtype=torch.float32)
    L = T
    q = x.q[L - 1:L].cuda()
    kc, vc = x.k[None].cuda(), x.v[None].cuda()
    do, dl = mimo.mimo_attn_decode(q, kc, vc, torch.tensor([L], dtype=torch.int32, device="cuda"),
                                   0, x.sinks.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (do[0] - po[L - 1]).abs().max().item() < 2e-3
    assert (dl[0] - pl[:, L - 1]).abs().max().item() < 1e-4


def test_ring_matches_linear_window():
    """A 129-slot ring holding the last 129 tokens equals the linear cache with window 129."""
    L = 1000
    x = W.prefill_inputs([L], hq=64, hkv=4, seed=22)
    ring_k = torch.empty((1, 129, 4, 192), dtype=torch.bfloat16)
    ring_v = torch.empty((1, 129, 4, 128), dtype=torch.bfloat16)
    for p in range(L - 129, L):
        ring_k[0, p % 129] = x.k[p]
        ring_v[0, p % 129] = x.v[p]
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    q = x.q[L - 1:L].cuda()
    a, la = mimo.mimo_attn_decode(q, ring_k.cuda(), ring_v.cuda(), sl, 129, x.sinks.cuda(),
                                  out_dtype=torch.float32)
    b, lb = mimo.mimo_attn_decode(q, x.k[None].cuda(), x.v[None].cuda(), sl, 129, x.sinks.cuda(),
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    # same keys, different order and split tiling: P is rounded to bf16 against
    # different running maxima, so the two agree to bf16 precision, not bitwise
    assert (a - b).abs().max().item() < 2e-3
    assert (la - lb).abs().max().item() < 1e-4
    ro, rl = oracle.decode(x.q[L - 1:L], x.k[None], x.v[None], [L], 129, x.sinks, ring=False)
    P.check(a, ro, la, rl, what="ring")


@pytest.mark.parametrize("window", [0, 129])
def test_full_caches(window):
    """Sequences that fill their linear cache to the last slot (L == capacity),
    and one slot short of it, under a multi-split plan."""
    lengths = [65536, 65535, 1, 40000]
    x = W.decode_inputs(lengths, 65536, window, seed=31 + window, device="cuda")
    out, lse = mimo.mimo_attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, window, x.sinks,
                                     out_dtype=torch.float32)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, window, x.sinks)
    P.check(out, ro, lse, rl, what=f"full caches W={window}")


def test_full_size_decode_global_and_ring():
    """Batch 64, lengths ~U[1024, 262144] in 262144-slot caches, and the 129-slot ring layer."""
    lengths = W.decode_b64_lengths(0)
    x = W.decode_inputs(lengths, W.DECODE_GA_CAPACITY, 0, seed=0, device="cuda")
    out, lse = mimo.mimo_attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    mimo.mimo_attn_device_status()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    Ls = np.array(lengths)
    pick = sorted({int(np.argmax(Ls)), int(np.argmin(Ls)), 0, 17, 63})
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks, batch_index=pick)
    idx = torch.as_tensor(pick, device="cuda")
    P.check(out[idx], ro, lse[idx], rl, what="GA decode b64")
    del x
    torch.cuda.empty_cache()
    r = W.decode_inputs(lengths, 129, 129, seed=1, device="cuda")
    out, lse = mimo.mimo_attn_decode(r.q, r.k_cache, r.v_cache, r.seqlens, 129, r.sinks)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.decode(r.q, r.k_cache, r.v_cache, r.seqlens, 129, r.sinks)
    P.check(out, ro, lse, rl, what="SWA ring decode b64")
