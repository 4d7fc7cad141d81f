"""Decode-step rotation + cache append (mimo_attn_rope_append) vs the fp64 oracle.

Rotated values are compared within the bf16 rounding of the output
(2^-8 relative, with a 1e-5 floor); the value slot and every untouched cache
slot are compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle.rope import append_slot, rope_append
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def _close(got, ref, what):
    g = P.to64(got)
    err = np.abs(g - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5
    assert np.all(err <= bound), f"{what}: worst {np.max(err - bound):.3e}"


def _new_token(B, hq=64, hkv=4, seed=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, hq, 192), generator=g).to(torch.bfloat16)
    k = torch.randn((B, hkv, 192), generator=g).to(torch.bfloat16)
    v = torch.randn((B, hkv, 128), generator=g).to(torch.bfloat16)
    return q, k, v


def _run(lengths, cap, window, theta, rotary_dim, seed):
    x = W.decode_inputs(lengths, cap, window, seed=seed, poison=False)
    q, kn, vn = _new_token(len(lengths), seed=seed + 1)
    rq, rk, rv = rope_append(q, kn, vn, x.k_cache, x.v_cache, x.seqlens, window, theta, rotary_dim)
    qd, knd, vnd = q.cuda(), kn.cuda(), vn.cuda()
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.cuda()
    mimo.mimo_attn_rope_append(qd, knd, vnd, kc, vc, sl, window, theta, rotary_dim)
    mimo.mimo_attn_device_status()
    return x, qd, kc, vc, rq, rk, rv


@pytest.mark.parametrize("window,cap,lengths", [
    (0, 8192, [1, 2, 100, 4097, 8192]),       # linear, full cache included
    (129, 129, [1, 128, 129, 130, 1000]),     # ring: wraps past the capacity
    (129, 4096, [1, 200, 4096]),              # linear cache with a window
])
@pytest.mark.parametrize("theta,rotary_dim", [(10000.0, 192), (1.0e6, 64), (500.0, 60)])
def test_rotation_and_append_match_oracle(window, cap, lengths, theta, rotary_dim):
    x, qd, kc, vc, rq, rk, rv = _run(lengths, cap, window, theta, rotary_dim, seed=cap + window)
    _close(qd, rq, "q")
    ring = window > 0 and cap == window
    kc0, vc0 = x.k_cache, x.v_cache
    kcg, vcg = kc.cpu(), vc.cpu()
    for b, L in enumerate(lengths):
        slot = append_slot(L, cap, ring)
        keep = torch.ones(cap, dtype=torch.bool)
        keep[slot] = False
        assert torch.equal(kcg[b, keep].view(torch.int16), kc0[b, keep].view(torch.int16))
        assert torch.equal(vcg[b, keep].view(torch.int16), vc0[b, keep].view(torch.int16))
        _close(kcg[b, slot], rk[b, slot], f"k slot b={b}")
        assert torch.equal(vcg[b, slot].double(), torch.from_numpy(rv[b, slot]))


def test_large_positions_keep_the_angle_accurate():
    """Position 262143: the angles are formed in double precision."""
    cap = 262144
    lengths = [cap, cap - 77]
    x = W.decode_inputs(lengths, cap, 0, hq=16, hkv=1, seed=40, poison=False)
    q, kn, vn = _new_token(2, hq=16, hkv=1, seed=41)
    rq, rk, _ = rope_append(q, kn, vn, x.k_cache, x.v_cache, x.seqlens, 0, 10000.0, 192)
    qd = q.cuda()
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    mimo.mimo_attn_rope_append(qd, kn.cuda(), vn.cuda(), kc, vc, x.seqlens.cuda(), 0, 10000.0, 192)
    mimo.mimo_attn_device_status()
    _close(qd, rq, "q at 262143")
    for b, L in enumerate(lengths):
        _close(kc[b, L - 1].cpu(), rk[b, L - 1], "k at large position")


def test_invalid_lengths_are_recorded_and_skipped():
    x = W.decode_inputs([5, 9], 8, 0, hq=4, hkv=1, seed=3, poison=False)
    q, kn, vn = _new_token(2, hq=4, hkv=1, seed=4)
    sl = torch.tensor([0, 9], dtype=torch.int32, device="cuda")  # L=0, and L > C on a linear cache
    qd, kc = q.cuda(), x.k_cache.cuda()
    mimo.mimo_attn_rope_append(qd, kn.cuda(), vn.cuda(), kc, x.v_cache.cuda(), sl, 0, 10000.0, 192)
    with pytest.raises(mimo.MimoAttnError) as e:
        mimo.mimo_attn_device_status()
    assert e.value.status == mimo.MIMO_ERR_INVALID_ARG
    assert torch.equal(qd.cpu().view(torch.int16), q.view(torch.int16))
    assert torch.equal(kc.cpu().view(torch.int16), x.k_cache.view(torch.int16))


@pytest.mark.parametrize("window,cap", [(0, 4096), (129, 129)])
def test_append_then_decode_matches_oracle(window, cap):
    lengths = [1, 64, 129, 130, 3000] if cap > 129 else [1, 64, 129, 130, 3000]
    x, qd, kc, vc, rq, rk, rv = _run(lengths, cap, window, 10000.0, 192, seed=77)
    sinks = x.sinks.cuda()
    out, lse = mimo.mimo_attn_decode(qd, kc, vc, x.seqlens.cuda(), window, sinks,
                                     out_dtype=torch.float32)
    mimo.mimo_attn_device_status()
    # the decode consumes the rotated query and key as stored (bf16); the
    # rotation's own rounding is checked above, so the oracle gets the same
    # stored values
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)  # noqa: E731
    ro, rl = oracle.decode(bf(rq), bf(rk), bf(rv), x.seqlens, window, x.sinks)
    P.check(out, ro, lse, rl, what=f"append+decode W={window} C={cap}")
