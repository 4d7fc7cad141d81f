"""FP8 (e4m3) KV-cache decode vs the fp64 oracle, through the C ABI.

The oracle decodes the same e4m3 codes from the format's definition and
applies the same per-KV-head scales, so the comparison isolates the kernel's
arithmetic (f16 products, fp32 accumulation, f16 P, bf16/fp32 output) from the
quantisation itself, with the tolerances of the bf16 path.
"""

import numpy as np
import pytest
import torch

import workloads as W
from oracle.fp8 import decode_fp8
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def run(x, out_dtype=torch.float32, v_scale=1.0, softmax_scale=None):
    d = lambda t: None if t is None else t.to("cuda")  # noqa: E731
    out, lse = mimo.mimo_attn_decode_fp8(d(x.q), d(x.k_codes), d(x.v_codes), d(x.k_scale),
                                         d(x.v_scale_kv), d(x.seqlens), x.window, d(x.sinks),
                                         out_dtype=out_dtype, v_scale=v_scale,
                                         softmax_scale=softmax_scale)
    mimo.mimo_attn_device_status()
    return out, lse


def ref(x, **kw):
    return decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, x.window,
                      x.sinks, **kw)


@pytest.mark.parametrize("window,capacity", [(0, 1024), (129, 1024), (129, 129), (1, 16), (0, 8192)])
@pytest.mark.parametrize("sinks", [True, False])
def test_small_batches(window, capacity, sinks):
    lengths = [1, 5, 64, 65, 130, 1000, 129, 128] if capacity >= 1000 else [1, 5, 16, 200, 129, 3]
    if capacity < 1000 and window == 1:
        lengths = [1, 2, 16, 9]
    if window == 0 or window != capacity:
        lengths = [min(L, capacity) for L in lengths]
    x = W.decode_inputs_fp8(lengths, capacity, window, hq=8, hkv=2, seed=capacity + window,
                            sinks=sinks)
    out, lse = run(x)
    ro, rl = ref(x)
    P.check(out, ro, lse, rl, what=f"fp8 W={window} C={capacity}")


def test_empty_sequence():
    x = W.decode_inputs_fp8([0, 7], 64, 0, hq=4, hkv=1, seed=3)
    out, lse = run(x)
    ro, rl = ref(x)
    P.check(out, ro, lse, rl, what="fp8 empty")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_model_heads(out_dtype):
    x = W.decode_inputs_fp8([3000, 17, 4097, 64, 65, 8191], 8192, 0, seed=9)
    out, lse = run(x, out_dtype)
    ro, rl = ref(x)
    P.check(out, ro, lse, rl, what=f"fp8 64/4 heads {out_dtype}")


def test_scales_and_overrides():
    """Non-default softmax scale and output scale, and distinct per-head cache scales."""
    x = W.decode_inputs_fp8([700, 2049, 33], 4096, 0, seed=14)
    assert len(set(x.k_scale.tolist())) == 4 and len(set(x.v_scale_kv.tolist())) == 4
    out, lse = run(x, v_scale=0.707, softmax_scale=0.05)
    ro, rl = ref(x, scale=0.05, v_scale=0.707)
    P.check(out, ro, lse, rl, what="fp8 scales")


def test_split_count_does_not_change_the_result():
    lengths = [5000, 300, 70]
    a = W.decode_inputs_fp8(lengths, 8192, 0, seed=12, poison=False)
    ro, rl = ref(a)
    for cap in (8192, 65536, 5000):
        k = torch.zeros((3, cap, 4, 192), dtype=torch.uint8)
        v = torch.zeros((3, cap, 4, 128), dtype=torch.uint8)
        n = min(cap, 8192)
        k[:, :n] = a.k_codes[:, :n]
        v[:, :n] = a.v_codes[:, :n]
        x = W.DecodeInputsFp8(a.q, k, v, a.k_scale, a.v_scale_kv, a.seqlens, a.sinks, 0, cap)
        out, lse = run(x)
        P.check(out, ro, lse, rl, what=f"fp8 split plan C={cap}")


def test_fp8_equals_bf16_decode_on_representable_values():
    """Caches whose values are exactly e4m3 codes times scales: the FP8 and bf16 paths see
    the same numbers and must agree to the rounding of P (f16 vs bf16)."""
    x = W.decode_inputs_fp8([1500, 129, 4000], 4096, 0, seed=17, poison=False)
    # power-of-two scales: code * scale is then exact in bf16 (4 significant bits of 8)
    # (the codes were drawn for scales near 2^-6, so these keep the values ~N(0, 1))
    x.k_scale = torch.tensor([2.0 ** -6, 2.0 ** -6, 2.0 ** -7, 2.0 ** -6])
    x.v_scale_kv = torch.tensor([2.0 ** -6, 2.0 ** -6, 2.0 ** -6, 2.0 ** -5])
    ks = x.k_scale.to(torch.float64).view(1, 1, -1, 1)
    vs = x.v_scale_kv.to(torch.float64).view(1, 1, -1, 1)
    kb = (x.k_codes.view(torch.float8_e4m3fn).to(torch.float64) * ks).to(torch.bfloat16)
    vb = (x.v_codes.view(torch.float8_e4m3fn).to(torch.float64) * vs).to(torch.bfloat16)
    assert torch.equal(kb.to(torch.float64), x.k_codes.view(torch.float8_e4m3fn).to(torch.float64) * ks)
    a, la = run(x)
    b, lb = mimo.mimo_attn_decode(x.q.cuda(), kb.cuda(), vb.cuda(), x.seqlens.cuda(), 0,
                                  x.sinks.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    # the bf16 path rounds P to 8 significant bits, the FP8 path to 11
    assert bool(((a - b).abs() <= 2e-3 + 2.0 ** -7 * b.abs()).all()), (a - b).abs().max().item()
    assert (la - lb).abs().max().item() < 1e-4


def test_full_size_decode_global_and_ring():
    """Batch 64, lengths ~U[1024, 262144] in 262144-slot e4m3 caches, and the 129-slot ring."""
    lengths = W.decode_b64_lengths(0)
    x = W.decode_inputs_fp8(lengths, W.DECODE_GA_CAPACITY, 0, seed=0, device="cuda")
    out, lse = mimo.mimo_attn_decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv,
                                         x.seqlens, 0, x.sinks)
    mimo.mimo_attn_device_status()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    Ls = np.array(lengths)
    pick = sorted({int(np.argmax(Ls)), int(np.argmin(Ls)), 0, 17, 63})
    ro, rl = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, 0,
                        x.sinks, batch_index=pick)
    idx = torch.as_tensor(pick, device="cuda")
    P.check(out[idx], ro, lse[idx], rl, what="fp8 GA decode b64")
    del x
    torch.cuda.empty_cache()
    r = W.decode_inputs_fp8(lengths, 129, 129, seed=1, device="cuda")
    out, lse = mimo.mimo_attn_decode_fp8(r.q, r.k_codes, r.v_codes, r.k_scale, r.v_scale_kv,
                                         r.seqlens, 129, r.sinks)
    mimo.mimo_attn_device_status()
    ro, rl = decode_fp8(r.q, r.k_codes, r.v_codes, r.k_scale, r.v_scale_kv, r.seqlens, 129,
                        r.sinks)
    P.check(out, ro, lse, rl, what="fp8 SWA ring decode b64")
